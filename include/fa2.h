/*
 * fa2.h -- C ABI of the B200 (sm_100a) exact-attention library libfa2.so.
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(Q K^T * scale [+ causal mask]) V
 *
 * tile by tile in on-chip memory, never writing an N x N matrix to HBM, and its
 * gradient by recomputing the probabilities from the saved log-sum-exp.
 *
 * Sources (page title, section):
 *   [DC]  "Flash Attention spiegata: una guida completa" (datacamp):
 *         "Attention standard vs Flash attention" (exact, not an approximation;
 *         tiles in fast on-chip memory, softmax applied incrementally);
 *         "Tiling"; "Ricomputazione" (the backward pass recomputes scores).
 *   [RU]  "FlashAttention-2" (systems-analysis.info wiki):
 *         "Предпосылки" (IO-aware tiling, memory linear in N);
 *         "Техническая архитектура и принципы работы" (fewer non-matmul
 *         operations, parallelism over the sequence, work split across warps).
 *   [QL]  "Flash Attention 2: attivarla (llama.cpp, Ollama, vLLM)" (qualellm.it):
 *         "Perché Flash Attention 2" (same mathematical result);
 *         troubleshooting "Errore unsupported head dimension" (unsupported head
 *         sizes are reported as an error).
 *
 * Conventions shared by every call
 *   - Tensors are dense, contiguous, row-major [B][H][N][d] in the 16-bit
 *     dtype given by ``dtype``; LSE and the backward's D are [B][H][N] float.
 *   - All pointers are DEVICE pointers on the current CUDA device, owned by the
 *     caller, 16-byte aligned.  The library keeps no reference after a call
 *     returns (work is enqueued on ``stream``).
 *   - ``causal`` = 1 lets query row i see keys 0..i; 0 lets it see all keys.
 *   - LSE_i = ln sum_j exp(S_ij) over the keys row i sees, S = scale * Q K^T.
 *   - The return value reports argument validation and launch only; the kernels
 *     run asynchronously.  Failures inside a kernel (a bounded wait that ran out)
 *     are reported by fa2_get_device_status().
 *   - Head dims: any multiple of 8 from 8 to 256 in the forward calls
 *     (fa2_fwd, fa2_fwd_window, fa2_fwd_decode), from 8 to 128 in the backward
 *     calls, and any multiple of 16 up to 128 in fa2_fwd_fp8.  Any other d
 *     returns FA2_ERR_UNSUPPORTED and launches nothing (no silent fallback).
 *   - Only compute capability 10.0 devices (B200, sm_100a) are supported;
 *     others return FA2_ERR_ARCH.
 *   - The library allocates one small device status word per device on first
 *     use and nothing per call.
 */
#ifndef FA2_H_
#define FA2_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* fa2_stream_t;

typedef enum {
  FA2_OK = 0,
  FA2_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size, flag or scale */
  FA2_ERR_UNSUPPORTED = 2, /* head dim the call does not support */
  FA2_ERR_ARCH = 3,        /* current device is not compute capability 10.0 */
  FA2_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  FA2_ERR_TIMEOUT = 5,     /* a bounded in-kernel wait ran out (device status) */
  FA2_ERR_WORKSPACE = 6    /* backward workspace null or too small */
} fa2_status;

typedef enum { FA2_FP16 = 0, FA2_BF16 = 1 } fa2_dtype;

/*
 * Forward pass.  [DC] "Tiling", "Attention standard vs Flash attention";
 * [RU] "Техническая архитектура и принципы работы".
 *
 *   Q, K, V : in,  [B][H][N][d] dtype
 *   O       : out, [B][H][N][d] dtype, O_i = sum_j softmax_j(S_i) V_j
 *   LSE     : out, [B][H][N] float (natural log, scaled-score units)
 *   B, H, N : >= 1; d a multiple of 8 up to 256; scale finite and > 0;
 *             causal in {0, 1};
 *   dtype   : FA2_FP16 or FA2_BF16
 * O must not overlap Q, K or V.  Results are bitwise repeatable run to run.
 */
int fa2_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
            int N, int d, float scale, int causal, int dtype, fa2_stream_t stream);

/*
 * Forward pass with a sliding window (local causal attention): query row i sees
 * keys max(0, i - window + 1) .. i, its ``window`` most recent keys.  Source:
 * [QL] "Modelli con attenzione a finestra scorrevole non standard" (models with
 * sliding-window attention, e.g. alternating local and global layers).
 *
 *   window : >= 1 (FA2_ERR_INVALID_ARG otherwise); window >= N is plain causal
 * Other arguments, layouts and errors as for fa2_fwd (causal is implied).  Key
 * tiles entirely outside a query tile's window are skipped, not masked.
 */
int fa2_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                   int H, int N, int d, float scale, int window, int dtype, fa2_stream_t stream);

/*
 * Decode-like forward: Nq query rows against Nk >= Nq key/value rows, e.g. one
 * new token (Nq = 1) against a long cache.  Source: [DC] "Parallelismo lungo la
 * lunghezza della sequenza" (with small batches and long sequences the batch x
 * heads grid leaves the GPU idle, so the work is also split along the
 * sequence).  The queries are the LAST Nq positions of the sequence: with
 * causal = 1 query i sees keys 0 .. Nk - Nq + i (bottom-right alignment; Nq = Nk
 * is fa2_fwd's causal mask); with causal = 0 every key.
 *
 * The key tiles (128 keys each) are cut into n_splits stretches; each stretch
 * is one CTA per 256 query rows per (batch, head).  With Nq <= 32 (<= 64) the
 * queries are also replicated 4 (2) times down the CTA's 128-row tile and each
 * copy scores a quarter (half) of every key tile's columns, so that four
 * softmax warps share the work of one query.  Each (stretch, copy) writes a
 * float partial output and log-sum-exp to the workspace and a second kernel
 * merges them (M = max_s L_s, O = sum_s e^{L_s - M} O_s / sum_s e^{L_s - M},
 * LSE = M + ln sum_s e^{L_s - M}).  One stretch and Nq > 64 write O and LSE
 * directly, like fa2_fwd.
 *
 *   Q, O     : [B][H][Nq][d] dtype (in, out)
 *   K, V     : [B][H][Nk][d] dtype (in)
 *   LSE      : out, [B][H][Nq] float
 *   B, H     : >= 1; 1 <= Nq <= Nk; d a multiple of 8 up to 256; causal in {0, 1}
 *   n_splits : 1 .. 1024 (FA2_ERR_INVALID_ARG otherwise); counts above the
 *              number of key tiles act as one tile per split
 *   workspace: device scratch of at least fa2_fwd_decode_workspace_size()
 *              bytes, 256-byte aligned, not overlapping any tensor argument
 *              (FA2_ERR_WORKSPACE otherwise); may be NULL when that size is 0.
 * Results are bitwise repeatable for a fixed n_splits; different split counts
 * round differently (within the stated tolerances).
 */
int fa2_fwd_decode(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                   int H, int Nq, int Nk, int d, float scale, int causal, int dtype, int n_splits,
                   void* workspace, size_t workspace_bytes, fa2_stream_t stream);

/*
 * Query tiles (128 rows) per CTA that fa2_fwd (window = 0) or fa2_fwd_window
 * uses for these sizes on a GPU with ``sm_count`` SMs (<= 0: the current
 * device's count): 2 (the softmax of one tile overlaps the other's products), or
 * 1 (twice the CTAs) for a causal call without a window whose two-tile grid,
 * ceil(N / 256) x B x H CTAs, is under one wave, or any other call whose one-tile
 * grid fits in one wave; always 1 for head dims above 128.  The test hook
 * fa2_debug_set_fwd_tiles overrides it.  Returns 0 for sizes fa2_fwd rejects, or
 * when sm_count <= 0 and no device can be queried.  Results do not depend on it.
 */
int fa2_fwd_tiles_per_cta(int B, int H, int N, int d, int causal, int window, int sm_count);

/*
 * The split count fa2_fwd_decode would best use for these sizes on a GPU with
 * ``sm_count`` SMs (<= 0: the current device's count): as many as keep all CTAs
 * in one wave (one CTA per SM, ceil(Nq / 256) x B x H CTAs per split), but no
 * more than one split per 4 key tiles, and at least 1.  Returns 0 for sizes
 * fa2_fwd_decode rejects, or when sm_count <= 0 and no device can be queried.
 */
int fa2_fwd_decode_splits(int B, int H, int Nq, int Nk, int d, int sm_count);

/*
 * Bytes of workspace fa2_fwd_decode needs with ``n_splits`` (0 when it writes O
 * and LSE directly, and for sizes or split counts fa2_fwd_decode rejects): float
 * partial outputs [S][B*H][Nq][d] and log-sum-exps [S][B*H][Nq], S the number of
 * non-empty stretches times the query copies (4 for Nq <= 32, 2 for Nq <= 64,
 * else 1), each part padded to 256 bytes.
 */
size_t fa2_fwd_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int n_splits);

/*
 * Forward pass with 8-bit (E4M3) inputs.  Source: [DC] FlashAttention-3 section
 * (FP8 attention: 8-bit floating point for the two matrix products).
 *
 *   Q, K, V : in,  [B][H][N][d] E4M3 bytes (1 sign, 4 exponent bits with bias 7,
 *             3 mantissa bits, no infinities), holding the real values
 *             q_scale * Q, k_scale * K, v_scale * V respectively
 *   O       : out, [B][H][N][d] bf16, softmax(scale * (q_scale Q)(k_scale K)^T) (v_scale V)
 *   LSE     : out, [B][H][N] float, in units of the scaled scores
 *   d       : a multiple of 16 from 16 to 128 (FA2_ERR_UNSUPPORTED otherwise)
 *   q_scale, k_scale, v_scale : finite and > 0 (per-tensor dequantisation scales)
 * Both products run on the 8-bit tensor cores (tcgen05 kind::f8f6f4) with fp32
 * accumulation; the probabilities P are rounded to E4M3 (relative error <= 2^-4,
 * absolute <= 2^-10 below 2^-6) before P V, and the row sums use the unrounded
 * values.  causal, B, H, N, scale and the errors as for fa2_fwd.
 */
int fa2_fwd_fp8(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
                int N, int d, float scale, int causal, float q_scale, float k_scale,
                float v_scale, fa2_stream_t stream);

/*
 * Bytes of device workspace fa2_bwd needs for these sizes (the per-row
 * D = rowsum(dO * O) and LSE * log2 e, a 256-byte counter that hands out the
 * key tiles, and a float32 dQ accumulator), a multiple of 256.
 * Returns 0 for sizes fa2_bwd would reject.
 */
size_t fa2_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass.  [DC] "Ricomputazione": the probabilities are recomputed from
 * Q, K and the saved LSE, then dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
 * dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q.
 *
 *   Q, K, V, O, dO : in,  [B][H][N][d] dtype (O and LSE as fa2_fwd wrote them)
 *   LSE            : in,  [B][H][N] float
 *   dQ, dK, dV     : out, [B][H][N][d] dtype
 *   d              : a multiple of 8 up to 128 (FA2_ERR_UNSUPPORTED otherwise)
 *   workspace      : scratch of at least fa2_bwd_workspace_size() bytes,
 *                    256-byte aligned, owned by the caller; its contents on
 *                    entry do not matter and on return are unspecified
 * Other arguments as for fa2_fwd.  dQ is accumulated with float atomics, so it
 * may differ in the last bits from run to run; dK and dV are repeatable (see
 * fa2_bwd_ex with FA2_BWD_DETERMINISTIC for a bitwise repeatable dQ).
 */
int fa2_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
            const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
            size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
            int dtype, fa2_stream_t stream);

/*
 * Backward of fa2_fwd_window: same window reading as the forward; arguments,
 * workspace and errors as for fa2_bwd (causal implied).  O and LSE must come
 * from fa2_fwd_window with the same window.
 */
int fa2_bwd_window(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                   const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                   size_t workspace_bytes, int B, int H, int N, int d, float scale, int window,
                   int dtype, fa2_stream_t stream);

/* Flags of fa2_bwd_ex. */
enum { FA2_BWD_DETERMINISTIC = 1 };

/*
 * Backward pass with options: the sliding window of fa2_bwd_window (window >= 1,
 * causal = 1; 0 = no window) and ``flags``:
 *
 *   FA2_BWD_DETERMINISTIC  dQ, dK and dV bitwise repeatable run to run.  Source:
 *     [RU] "Производительность и эффективность" (the method stays exact and
 *     deterministic).  dQ is then computed by a query-stationary kernel that
 *     recomputes the scores and dP and sums dQ over the key tiles in tensor memory
 *     in a fixed order, instead of adding key-tile partials into a float
 *     accumulator in global memory (whose order of addition varies); dK and dV
 *     come from a kernel without the dQ product.  Seven matrix products per tile
 *     pair instead of five, on 128-wide tiles at every head dim: measured on B200
 *     about 7 % slower than the default at d = 128, about twice the time at d = 64.
 *     The workspace holds only the two per-row statistics and the tile counter.
 *
 * Arguments, layouts, results and errors otherwise as fa2_bwd (and
 * fa2_bwd_window); flags other than FA2_BWD_DETERMINISTIC, window < 0 or a window
 * with causal = 0 return FA2_ERR_INVALID_ARG.  The workspace must hold
 * fa2_bwd_ex_workspace_size(B, H, N, d, flags) bytes.
 */
int fa2_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
               const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
               size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
               int window, int flags, int dtype, fa2_stream_t stream);

/* Bytes of workspace fa2_bwd_ex needs with ``flags`` (0 for sizes or flags it
 * rejects); without flags, fa2_bwd_workspace_size. */
size_t fa2_bwd_ex_workspace_size(int B, int H, int N, int d, int flags);

/*
 * Allocation-free backward.  The paper has no counterpart: this entry point
 * exists for callers that cannot call cudaMalloc -- runtimes that hand out device
 * memory only from their own fixed pool, and latency-critical code that must not
 * take the device-wide synchronisation an allocation can cause -- and so cannot
 * provide the workspace fa2_bwd asks for.
 *
 * Same arguments, results and errors as fa2_bwd, minus the workspace: the
 * scratch lives in a 32 MiB buffer that the library holds in device memory on
 * every GPU that loads it, until the process exits.  Nothing is allocated.
 *   - Sizes whose workspace (fa2_bwd_workspace_size) exceeds 32 MiB - 256 bytes
 *     return FA2_ERR_WORKSPACE and launch nothing (e.g. B*H = 64, N = 1024,
 *     d = 64 fits; B*H = 128, N = 4096, d = 128 does not).
 *   - The first call on a device looks up the buffer's device address (set-up);
 *     make that first call before any stream capture.
 *   - Every call shares the one buffer and it keeps the last call's contents;
 *     each call rewrites all of it that it reads (the dQ accumulator is zeroed
 *     by the call itself).  Calls that overlap on the GPU -- on different
 *     streams, or from several host threads -- race on the buffer and give
 *     wrong results: serialise them.
 *   - In-kernel wait timeouts go to a status word in the first 256 bytes of the
 *     buffer; fa2_get_device_status() reads and clears it with the library's
 *     own word and allocates nothing, so a caller that only ever uses this entry
 *     point sees its timeouts there too.
 */
int fa2_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                    float scale, int causal, int dtype, fa2_stream_t stream);

/*
 * Synchronises ``stream``, then returns and clears the current device's status
 * words (the library's, and fa2_bwd_noalloc's if that call has run on the
 * device): FA2_OK, or FA2_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last call (the kernel then skipped its output and exited cleanly; the CUDA
 * context stays usable).  FA2_ERR_CUDA if the synchronisation itself failed.
 * If ``site`` is not NULL it receives the id of the wait that ran out (0 if none).
 * Allocates nothing.  (``site`` is one argument more than a bare status query
 * needs; it tells which wait of which kernel ran out.)
 */
int fa2_get_device_status(fa2_stream_t stream, int* site);

/* Human-readable name of a status code (static storage). */
const char* fa2_status_string(int status);

/*
 * Test hook.  ``wait_limit_ms`` sets the wall-clock budget of every bounded
 * in-kernel wait (0 restores the default of 2000 ms).  ``fault`` = 1 makes the
 * next forward launches skip their first K-tile load and the next backward
 * launches skip their K and V load, so a consumer's wait runs out and the
 * timeout path is exercised without any GPU fault; 0 turns it off.  Not for
 * production use.
 */
void fa2_debug_set(int fault, unsigned int wait_limit_ms);

/*
 * Test hook.  Caps the backward's persistent grid at ``max_ctas`` CTAs (0, the
 * default, restores one CTA per SM), so that small problems run several key tiles
 * per CTA.  Results do not depend on it.  Not for production use.
 */
void fa2_debug_set_bwd_grid(int max_ctas);

/*
 * Test hook.  Query tiles (128 rows) per forward CTA for fa2_fwd and
 * fa2_fwd_window at head dims up to 128: 1 or 2 forces that many; 0, the default,
 * restores the library's choice (two, unless one fills the SMs better: causal
 * calls whose two-tile grid is under one wave, other calls whose one-tile grid
 * fits in one wave).  Results do not depend on it.  Not for production use.
 */
void fa2_debug_set_fwd_tiles(int tiles);

/* Number of kernels this library has launched in this process (all devices). */
unsigned long long fa2_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FA2_H_ */
