"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .fourier_oracle import (  # noqa: F401
    Hybrid,
    attention,
    basis,
    compress,
    decode,
    partition,
    reconstruct,
    split_dims,
)
