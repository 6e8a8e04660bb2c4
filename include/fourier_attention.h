/*
 * fourier_attention.h -- C ABI of the B200 (sm_100a) Fourier-approximated KV cache.
 *
 * The method (FourierAttention, arXiv 2506.11886): the head dimensions of a KV cache
 * that are insensitive to long context are projected, over the middle span of the
 * sequence, onto the first k functions of an orthonormal real Fourier basis; the first
 * S ("sink") tokens, the last R ("recent") tokens and the remaining head dimensions stay
 * exact. Decoding attends over this hybrid cache directly in the coefficient domain.
 *
 * Sources, cited by page title and section:
 *   [abstract] shd-paper.top summary of arXiv 2506.11886, "Beyond Homogeneous Attention:
 *              Memory-Efficient LLMs via Fourier-Approximated KV Cache", abstract and
 *              "method details".
 *   [skill]    agent-skills.jp "fourier-approximated-kv-cache" skill page: "Architecture
 *              overview", Step 2 (fourier_compress_kv_cache), Step 3
 *              (selective_preserve_tokens), Step 4 (reconstruct_from_fourier), "Practical
 *              guidance" (custom kernels for the memory-bound prefill/decode work).
 *
 * Conventions shared by every entry point
 *   - Head dimension D is fixed at 128. Query head h of batch row b reads KV head
 *     g = h / (Hq / Hkv) (grouped-query attention).
 *   - Every device pointer is caller-owned device memory (for example from PyTorch) and
 *     must be 16-byte aligned. The library never allocates device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     All work is enqueued asynchronously on it; host arguments are consumed before the
 *     call returns.
 *   - Return value: FA_OK, or an error code with a message in fa_last_error(). Argument
 *     errors are detected on the host before anything is launched. Nothing aborts the
 *     process.
 *   - bf16 = IEEE bfloat16 (round-to-nearest-even on every store); fp32 accumulation.
 */
#ifndef FOURIER_ATTENTION_H
#define FOURIER_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_HEAD_DIM 128
#define FA_MAX_KV_HEADS 64   /* KV heads per layer */
#define FA_MAX_K_DECODE 2047 /* largest k fa_decode supports */

enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID = 1,     /* bad argument: null/misaligned pointer, inconsistent shape */
  FA_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement (D != 128, ...) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  FA_ERR_DEVICE = 4       /* a kernel's bounded wait expired (see fa_device_status) */
};

enum fa_dtype { FA_BF16 = 0, FA_F32 = 1 };

/* Shape of one layer's cache. B batch rows, Hq query heads, Hkv KV heads (Hq % Hkv == 0),
 * D = 128, L cached tokens, S sink and R recent tokens kept exact, k basis functions. */
typedef struct fa_shape {
  int32_t B, Hq, Hkv, D, L, S, R, k;
} fa_shape;

/*
 * fa_plan: everything derived on the host from (shape, dim mask); plain data, no pointers.
 *
 * Token partition ([skill] Step 3): sink [0, S), middle [S, S + M), recent [L - R, L),
 * each token in exactly one part. If L <= S + R the middle is empty (M = 0) and the
 * sink/recent windows shrink so that they cover the L tokens once: S = min(S, L),
 * R = min(R, L - S).
 *
 * Dim split ([abstract]: only the long-context-insensitive dims are projected): for KV
 * head g, perm[g][0 .. dc[g]) lists the compressed dims in ascending order and
 * perm[g][dc[g] .. 128) the retained dims in ascending order.
 *
 * Basis period P: the middle span is projected onto the first k functions of the
 *   orthonormal real Fourier basis of period P. fa_plan_init sets P = M. A cache that
 *   takes appended tokens while decoding (fa_append) is planned with room for them
 *   (fa_plan_reserve): P = L_max - S - R >= M stays fixed while M grows, and the middle
 *   tokens t < M are projected onto the period-P functions, which equals projecting the
 *   middle zero-padded to P tokens. (The pages give fixed-length spectral coefficients
 *   and a recent window of the current sequence; they do not say how the cache is kept
 *   while decoding. This is the reading the library takes.)
 *
 * Hybrid cache layout (element offsets; F and E bf16, C fp32):
 *   F (sink + recent rows, all dims): [B][Hkv][S + R][128]; row i < S is token i, and
 *     the recent rows form a ring: row S + ((recent_head + i) mod R) is token L - R + i
 *     (recent_head = 0 until fa_append advances it).
 *   E (middle rows, retained dims), room for P rows: element (b, g, t, i) of middle
 *     token t < M and retained
 *     dim i < de_ld[g] sits at b * e_batch + e_off[g] + t * e_pitch[g] + i; columns
 *     [de[g], de_ld[g]) are zero. Two arrangements:
 *     e_token_major = 0: one dense [P][de_ld[g]] block per KV head (e_pitch[g] = de_ld[g],
 *       de_ld[g] = de[g] rounded up to a multiple of 8, blocks in KV-head order);
 *     e_token_major = 1: the rows of all KV heads of a batch interleaved per token, so
 *       that token t of batch b is one contiguous row of Hkv * w elements (de_ld[g] = w
 *       for every g, e_off[g] = g * w, e_pitch[g] = Hkv * w, w = 8, 16 or 32, the
 *       smallest that holds every de[g]; w = 0 when every dim is compressed).
 *     fa_plan_init chooses token-major exactly when fa_decode will run the middle span on
 *     the tensor cores: middle span present, k <= 255, G in {1, 2, 4}, every de[g] <= 32,
 *     either k * G >= 255 and B * Hq >= 128, or B * Hq >= 1024 (a warp then reads one
 *     token's retained dims of 32 query heads as one coalesced row).
 *   C (Fourier coefficients of the middle rows, compressed dims, fp32): block of (b, g)
 *     starts at b * c_batch + c_off[g] and is [kk][dc_ld[g]] row-major,
 *     kk = (M > 0 ? k : 0); columns [dc[g], dc_ld[g]) are zero. Row j is basis function j.
 *     C is kept in fp32: it holds k * dc values per head against M * de for E (about 2%
 *     of the cache at k = M / 128), and a bf16 C would add a second rounding of up to
 *     2^-8 relative to every reconstructed value.
 * dc_ld is dc rounded up to a multiple of 8 (rows of 32 bytes).
 *
 * Basis table (fa_build_basis) row stride: phi_ld = P rounded up to a multiple of 8.
 */
typedef struct fa_plan {
  fa_shape shape;
  int32_t S, R, M, kk, G;
  int32_t phi_ld;
  int32_t e_token_major;
  int32_t P;           /* basis period, P >= M (P = M = 0 without a middle span) */
  int32_t recent_head; /* ring position of the oldest recent row, 0 <= recent_head < max(R, 1) */
  int32_t dc[FA_MAX_KV_HEADS], de[FA_MAX_KV_HEADS];
  int32_t dc_ld[FA_MAX_KV_HEADS], de_ld[FA_MAX_KV_HEADS];
  int32_t e_pitch[FA_MAX_KV_HEADS];
  int64_t c_off[FA_MAX_KV_HEADS], e_off[FA_MAX_KV_HEADS];
  int64_t c_batch, e_batch;
  int64_t f_elems, e_elems, c_elems; /* elements of each of F_K/F_V, E_K/E_V, C_K/C_V */
  uint8_t perm[FA_MAX_KV_HEADS][FA_HEAD_DIM];
} fa_plan;

/* The hybrid cache of one layer: six caller-allocated device buffers sized by the plan
 * (f_elems, e_elems, c_elems): F_K, F_V, E_K, E_V bf16; C_K, C_V fp32. This is the dict
 * {initial, recent, middle_compressed} of [skill] Step 3, with the retained dims of the
 * middle (E) kept beside the coefficients (C). */
typedef struct fa_cache {
  void* F_K;
  void* F_V;
  void* E_K;
  void* E_V;
  void* C_K;
  void* C_V;
} fa_cache;

/*
 * fa_plan_init -- derive the plan of one layer.
 *   shape     host pointer; D must be 128, 1 <= Hkv <= FA_MAX_KV_HEADS, Hq % Hkv == 0,
 *             B >= 1, L >= 1, S >= 0, R >= 0, k >= 1. If the middle is non-empty and
 *             some dim is compressed, k <= M is required.
 *   dim_mask  host uint8 [Hkv][128]; nonzero = that dim of that KV head is compressed.
 *   plan      host output, fully written on success.
 * Returns FA_ERR_INVALID / FA_ERR_UNSUPPORTED for shapes the rules above reject.
 * Pure host function; touches no device.
 */
int fa_plan_init(const fa_shape* shape, const uint8_t* dim_mask, fa_plan* plan);

/*
 * fa_plan_reserve -- make room in a plan for tokens appended while decoding (fa_append).
 *   plan   host, in/out: a plan from fa_plan_init with a middle span (M >= 1) and nothing
 *          reserved or appended yet (P == M). On success P = L_max - S - R, phi_ld and
 *          every layout field are re-derived (E holds P rows per KV head), and the plan
 *          accepts up to L_max - L calls of fa_append. Call it before allocating the
 *          cache and before fa_build_basis / fa_compress, which then use period P.
 *   L_max  largest sequence length the cache will hold, L <= L_max, L_max - S - R < 2^21.
 * Returns FA_ERR_INVALID (bad plan or L_max) or FA_ERR_UNSUPPORTED (no middle span, or a
 * plan already reserved / appended to). Pure host function.
 */
int fa_plan_reserve(fa_plan* plan, int32_t L_max);

/*
 * fa_build_basis -- the orthonormal real Fourier basis over a span of M tokens, transposed.
 * ([abstract] "orthogonal Fourier bases"; [skill] Step 2 keeps the leading spectral
 * terms of a real FFT along the sequence.) M is the basis period: pass the plan's P (which
 * equals the middle length unless fa_plan_reserve made room).
 *   phi_0(t) = 1/sqrt(M); for j >= 1, f = (j + 1) / 2 and phi_j is sqrt(2/M) cos(2 pi f t / M)
 *   (j odd) or sqrt(2/M) sin(2 pi f t / M) (j even); the cosine at f = M/2 (M even) uses
 *   1/sqrt(M). The phase f*t is reduced modulo M exactly in integers first.
 *   normalized = 1: phiT[j * ld + t] = phi_j(t).
 *   normalized = 0: the same functions without their scale (1 for DC, cos / sin of unit
 *                   amplitude otherwise). This is the table fa_compress reads (dtype
 *                   FA_BF16): the scales are applied in fp32 after accumulation, so the
 *                   DC and Nyquist rows are exact in bf16 and no constant rounding error
 *                   of 1/sqrt(M) or sqrt(2/M) biases the coefficients.
 *   Columns [M, ld) are written as 0. dtype FA_BF16 or FA_F32. Requires 1 <= k <= M,
 *   ld >= M, ld a multiple of 8. phiT: device, k * ld elements.
 */
int fa_build_basis(int32_t M, int32_t k, int32_t dtype, int32_t normalized, void* phiT,
                   int64_t ld, void* stream);

/*
 * fa_compress -- prefill compression of one layer ([skill] Steps 2-3; [abstract]).
 *   K, V   device bf16 [B][Hkv][L][128], the full-precision cache (read only).
 *   phiT   device bf16 [k][plan->phi_ld] from fa_build_basis(P, k, FA_BF16, 0, ...) (the
 *          unscaled table of period P; columns t < M are read); may be NULL only when
 *          M == 0.
 *   cache  host struct of device output buffers (see fa_plan for layouts); written:
 *          F = sink/recent rows, E = retained dims of the middle (bit-exact copies),
 *          C = Phi^T X[S:S+M, compressed dims], fp32 (bf16 x bf16 products accumulated in
 *          fp32 on the tensor cores, then scaled by the orthonormal factor of each row);
 *          the recent rows go to F in the ring order of plan->recent_head.
 * The projection runs on the tcgen05 tensor cores (TMA-fed, accumulator in TMEM).
 * Requires bf16 values to be finite (a non-finite recent-token value meets a zero basis
 * entry in the ragged last K tile).
 */
int fa_compress(const fa_plan* plan, const void* K, const void* V, const void* phiT,
                const fa_cache* cache, void* stream);

/*
 * fa_decode_workspace_size -- bytes of scratch fa_decode needs for `num_splits` split-L
 * partitions of the middle span (num_splits <= 0: the automatic choice fa_decode makes
 * for the current device). Returns 0 if the plan is unusable for decode.
 */
size_t fa_decode_workspace_size(const fa_plan* plan, int32_t num_splits);

/*
 * fa_decode_describe -- how fa_decode would run a plan (no counterpart in the paper; a
 * host-side query for callers that size launches, graphs or profiles).
 *   info->split_kernel  which kernel runs the middle span (enum fa_split_kernel);
 *   info->num_splits    split-L partitions (num_splits <= 0: the automatic choice for the
 *                       current device, as fa_decode makes it);
 *   info->cluster       CTAs per thread-block cluster of the split kernel (1 = no cluster);
 *   info->launches      kernels one fa_decode call launches.
 * Returns the status fa_decode_workspace_size would imply (message in fa_last_error()).
 */
enum fa_split_kernel {
  FA_SPLIT_NONE = 0,        /* no middle span: only the sink / recent rows */
  FA_SPLIT_CUDA_CORES = 1,  /* fp32 CUDA-core split kernel */
  FA_SPLIT_TC_TOKEN_MAJOR = 2, /* tcgen05 split kernel over token-major E (k <= 255) */
  FA_SPLIT_WARP_MMA = 3,    /* warp-level MMA split kernel (256 <= k <= 1023) */
  FA_SPLIT_TC_CLUSTER = 4   /* tcgen05 split kernel, coefficient slots split over a cluster
                               (256 <= k <= 1023, G in {2, 4, 8}, B * Hq filling its sets of
                               128 query heads at least three quarters; else warp MMA) */
};
typedef struct fa_decode_info {
  int32_t split_kernel, num_splits, cluster, launches;
} fa_decode_info;
int fa_decode_describe(const fa_plan* plan, int32_t num_splits, fa_decode_info* info);

/*
 * fa_decode -- one decode step: every query attends to all L tokens of the hybrid cache.
 * ([skill] Step 4, restore during decoding; [abstract].)
 *   q     device bf16 [B][Hq][128], one query per sequence and head.
 *   cache the hybrid cache written by fa_compress with the same plan.
 *   out   device [B][Hq][128] of out_dtype: FA_F32, or FA_BF16 (the fp32 result rounded to
 *         nearest even).
 * Scores of the compressed dims are Phi (C_K q_c) and their values (Phi^T p) C_V, with the
 * basis regenerated in-kernel (sincos recurrence), never read from memory; the exact dims,
 * sink and recent tokens use plain dot products. Softmax scale 1/sqrt(128); fp32 online
 * softmax across split-L partitions merged by a combine pass. The result equals softmax
 * attention over the reconstructed cache (Phi C on the compressed dims of the middle).
 *   workspace  device scratch of at least fa_decode_workspace_size(plan, num_splits) bytes.
 * The basis of the middle span has period P (fa_plan_reserve); tokens t < M are read.
 * Requires k <= FA_MAX_K_DECODE and P < 2^21 tokens.
 */
int fa_decode(const fa_plan* plan, const void* q, const fa_cache* cache, void* out,
              int32_t out_dtype, void* workspace, size_t workspace_bytes, int32_t num_splits,
              void* stream);

/*
 * fa_decode_noalloc -- fa_decode for callers that cannot allocate device memory.
 * (The paper has no counterpart; this is a deployment convenience of this library.)
 *   Some callers cannot call cudaMalloc or hand over scratch memory: plug-ins running
 *   inside a host framework that owns every device allocation and exposes no allocator
 *   to them, serving loops that carved all of HBM into their own pools at start-up, and
 *   latency-critical paths that must not take the implicit device synchronisation of
 *   cudaMalloc / cudaFree. This entry point needs no workspace argument: its scratch is a
 *   fixed array of FA_NOALLOC_SCRATCH_BYTES inside the library's device image, which
 *   every GPU that loads the library holds until the process exits.
 *   Arguments are those of fa_decode without workspace / workspace_bytes. num_splits <= 0
 *   picks the split count fa_decode would pick, lowered until the scratch fits; a given
 *   num_splits is used as is. If the scratch cannot hold even one split, the call
 *   returns FA_ERR_UNSUPPORTED (message gives the bytes needed) and launches nothing.
 *   Calls no cudaMalloc / cudaFree and no allocating library routine.
 *   Set-up: the first call on each device (with that device current) looks up the
 *   device address of the scratch array; make that first call before any stream
 *   capture begins. The address is kept per device and CUDA context: after
 *   cudaDeviceReset the next call looks it up again (in the new context), so that call
 *   too belongs before any capture.
 *   Errors: the plan checks and configuration limits of fa_decode, reported with their
 *   own message.
 *   All calls in the process share one scratch array per device and it keeps the last
 *   call's contents; the kernels write every scratch word before reading it, so nothing
 *   needs clearing. Calls whose kernels overlap on the same GPU (different streams, no
 *   ordering between them) race on the scratch and give wrong results.
 */
#define FA_NOALLOC_SCRATCH_BYTES (16u << 20)
int fa_decode_noalloc(const fa_plan* plan, const void* q, const fa_cache* cache, void* out,
                      int32_t out_dtype, int32_t num_splits, void* stream);

/*
 * fa_append -- add one token to every sequence of a compressed cache while decoding
 * (decode-time cache maintenance). The pages keep a recent window of the current
 * sequence ([skill] Step 3) and fixed-length spectral coefficients for the middle
 * ([abstract] method details); this entry point keeps both as the sequence grows.
 *   plan    host, in/out: a plan with room left (M < P, see fa_plan_reserve). On success
 *           the plan describes the longer sequence: L and M grow by 1 and recent_head
 *           advances by one ring position (when R > 0).
 *   k_new, v_new  device bf16 [B][Hkv][128]: the key and value of the new token L.
 *   cache   the hybrid cache written by fa_compress / fa_append under this plan.
 * Per (b, g): the oldest recent token x (the new token itself when R == 0) leaves the
 * recent window and becomes middle token t = M: its retained dims are written to E row t
 * (padding columns zero) and its compressed dims are folded into the coefficients,
 * C_j += phi_j(t) x_c for every j < k (the rank-1 update that extends the projection by
 * one token under the fixed period P, fp32). The new token takes the freed ring row.
 * The result equals fa_compress of the longer sequence with the same period, up to fp32
 * rounding of the coefficients (E and F are bit-exact).
 * Returns FA_ERR_UNSUPPORTED when no room is left (M == P) or the plan has no middle
 * span; argument errors as for the other entry points. Launches one kernel (two when the
 * fold is split into row chunks to fill the GPU). The position (t = M, the ring head) is
 * taken from the plan when the call is made, so a CUDA graph that captured this call
 * replays that same position.
 */
int fa_append(fa_plan* plan, const void* k_new, const void* v_new, const fa_cache* cache,
              void* stream);

/*
 * fa_dim_sensitivity -- head-dimension sensitivity scores, for choosing the dim mask of
 * fa_plan_init ([skill] Step 1 and "Architecture overview": a noise-perturbation analysis
 * finds the dims that must stay exact; the dims least sensitive to noise are compressed).
 *   shape   host; B, Hq, Hkv, D = 128 and L are used (S, R, k are ignored).
 *           Hq / Hkv in {1, 2, 4, 8}.
 *   q       device bf16 [B][Hq][128]: the probe queries.
 *   K       device bf16 [B][Hkv][L][128]: the keys (full precision, the layout of fa_compress).
 *   noise   device bf16 [B][Hkv][L][128]: N(0, 1) draws, one per token and dim (the
 *           caller's random numbers).
 *   scores  device fp32 [Hkv][128], written: scores[g][d] is the Frobenius norm, over every
 *           batch row, every query head of KV head g and every output dim, of the change of
 *           softmax attention (scale 1/sqrt(128)) when value dim d of every token of KV head
 *           g gets FA_NOISE_SCALE * noise added.
 * Only the values change, so the output change is FA_NOISE_SCALE * P n_d with P the
 * attention weights: the library runs one exact attention pass over (K, noise) and takes
 * per-dim norms. The values themselves are not needed and not read.
 *   workspace  device scratch of at least fa_dim_sensitivity_workspace_size(shape) bytes.
 * Returns 0 from the size query for unusable shapes.
 */
#define FA_NOISE_SCALE 0.1f
size_t fa_dim_sensitivity_workspace_size(const fa_shape* shape);
int fa_dim_sensitivity(const fa_shape* shape, const void* q, const void* K, const void* noise,
                       float* scores, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_select_dims -- host: the dim mask from sensitivity scores. For each KV head g the
 * n_compressed dims with the lowest scores[g][*] are marked compressed (1), the others
 * retained (0); equal scores rank by dim index. scores: host fp32 [Hkv][128]; mask_out:
 * host uint8 [Hkv][128], the dim_mask argument of fa_plan_init. Requires
 * 1 <= Hkv <= FA_MAX_KV_HEADS and 0 <= n_compressed <= 128. Pure host function.
 */
int fa_select_dims(const float* scores, int32_t Hkv, int32_t n_compressed, uint8_t* mask_out);

/*
 * fa_device_status -- synchronise `stream`, then read and clear the library's kernel
 * watchdog word. Returns FA_OK if no kernel launched since the last call hit a wait
 * limit, FA_ERR_DEVICE (message names the kernel and wait) if one did, FA_ERR_CUDA if
 * the stream reported an error. Kernels that hit a limit stop their work, release their
 * tensor memory and return instead of hanging.
 */
int fa_device_status(void* stream);

/*
 * fa_watchdog_selftest -- diagnostics for the bounded-wait path (no counterpart in the
 * paper). Launches one CTA whose thread waits on an mbarrier that nothing ever completes,
 * with a wall-time bound of `wait_ns` (1 us .. 1 s). The wait expires, the kernel records a
 * watchdog code and returns normally; the next fa_device_status(stream) must then report
 * FA_ERR_DEVICE and clear it. Nothing faults, traps or hangs.
 */
int fa_watchdog_selftest(uint32_t wait_ns, void* stream);

/* Message of the last non-FA_OK return on the calling thread ("" if none). */
const char* fa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FOURIER_ATTENTION_H */
