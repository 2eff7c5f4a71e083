/*
 * cswa_attn.h -- C ABI of the B200 (sm_100a) causal sliding-window GQA attention block.
 *
 * The operation is the causal self-attention of the nanochat GPT: queries and
 * keys RMS-normalised (no weight) and rotated by RoPE, grouped-query heads
 * (Hkv <= Hq, query head h reads KV head h / (Hq/Hkv)), and a per-layer causal
 * sliding window (nanochat Admin & Developer Guide, 3 "The GPT Model
 * (Internals)" and its "Sliding-window attention" part; 6 "Attention: FA3 with
 * SDPA Fallback"; 7 "KV cache"), with the plain softmax attention of the
 * nanoGPT Administrator & Developer Guide, 8 "CausalSelfAttention".
 *
 * Conventions shared by every call
 *   - Tensors are device memory owned by the caller. The library never
 *     allocates: where a call needs scratch space, the caller passes a
 *     workspace of at least the size the matching *_workspace_bytes() returns.
 *   - bf16 tensors are stored as raw 16-bit words, in BTHD layout: (B, T, H, D)
 *     contiguous, D fastest. Every tensor pointer must be 16-byte aligned.
 *   - D (head dim) is 64 or 128. Hq % Hkv == 0. B, T >= 1.
 *   - window W >= 0: key j is visible from query i iff 0 <= i - j <= W
 *     (W + 1 keys including the query itself; FlashAttention's (left=W,
 *     right=0)). W < 0: plain causal, no window. W >= T - 1 equals W < 0.
 *   - scale multiplies q.k (1/sqrt(D) for plain attention; nanochat's QK gain
 *     is folded in here). It must be finite and > 0.
 *   - lse is the natural-log log-sum-exp of the scaled scores, fp32.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous: they enqueue kernels and return.
 *   - Argument errors are reported synchronously, before anything is
 *     enqueued, and leave every output untouched. Errors found on the device
 *     (a wait that timed out, a decode position out of range) are recorded in a
 *     per-device status word that attn_get_status() returns and clears.
 *   - Calls on different streams may run concurrently; they share nothing but
 *     the status word.
 */
#ifndef CSWA_ATTN_H
#define CSWA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, Hq % Hkv != 0, bad scale */
  ATTN_ERR_UNSUPPORTED = 2, /* head dim other than 64/128, or not an sm_100 device */
  ATTN_ERR_LAUNCH = 3,      /* a CUDA launch or tensor-map encode failed */
  ATTN_ERR_TIMEOUT = 4,     /* a device-side wait gave up (reported by attn_get_status) */
  ATTN_ERR_DEVICE = 5       /* a device-side range check failed (reported by attn_get_status) */
} attn_status_t;

/*
 * attn_rope_qknorm -- the fused prologue (nanochat Admin & Developer Guide, 3):
 *   for every row x (D values) of q (B,T,Hq,D) and of k (B,T,Hkv,D):
 *     xh = x / sqrt(mean(x^2) + eps)
 *     (y_j, y_{j+D/2}) = rotation of (xh_j, xh_{j+D/2}) by phi_j = p * rope_base^(-2j/D)
 *   with p = t + (pos ? pos[b] : 0). v is not touched.
 * q/k may be null (then q_out/k_out are ignored), not both. q_out may equal q
 * and k_out may equal k (in place). pos: optional int32 device array (B).
 * eps >= 0, rope_base > 1.
 */
attn_status_t attn_rope_qknorm(const void* q, const void* k, void* q_out, void* k_out, const int32_t* pos,
                               int B, int T, int Hq, int Hkv, int D, float rope_base, float eps, void* stream);

/*
 * attn_rope_qknorm_bwd -- gradient of the prologue: given the raw q, k and the
 * gradients dq_hat, dk_hat with respect to its outputs, writes
 *   dx = (g - xh (g . xh) / D) / r,   r = sqrt(mean(x^2) + eps),
 * where g is dx_hat rotated by -phi. Same shapes, nullability and aliasing
 * rules as attn_rope_qknorm (dq may equal dq_hat).
 */
attn_status_t attn_rope_qknorm_bwd(const void* q, const void* k, const void* dq_hat, const void* dk_hat,
                                   void* dq, void* dk, const int32_t* pos, int B, int T, int Hq, int Hkv,
                                   int D, float rope_base, float eps, void* stream);

/*
 * attn_fwd -- o = softmax(scale * q k^T restricted to the causal window) v.
 *   q (B,T,Hq,D), k and v (B,T,Hkv,D) bf16 -> o (B,T,Hq,D) bf16, lse (B,Hq,T) fp32.
 * o and lse must not overlap the inputs. tcgen05 tensor cores, fp32 accumulation.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T,
                       int Hq, int Hkv, int D, int window, float scale, void* stream);

/* Bytes of workspace attn_bwd needs for this window: per query row, -lse/scale and
 * -Delta_i = -(dO_i . o_i) as bf16 hi/lo pairs (2 x B*Hq*Tpad*4 bytes, Tpad = T
 * rounded up to a multiple of 128); the bf16 dS^T tiles (128 x 128) of every (query
 * tile, key tile) pair inside the causal window, kept between the main backward
 * kernel and the dQ kernel: about B*Hq*T*min(T, W+128)*2 bytes for window W
 * (B*Hq*T^2 without a window); and 256 bytes for the work counters; each part
 * rounded up to 256 bytes. Nothing in it needs to be initialised. */
size_t attn_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int window);

/* The least workspace attn_bwd and attn_block_bwd accept: the row extensions, the
 * counters and the dS^T tiles of ONE (batch, KV head) block, i.e. about
 * (Hq/Hkv)*T*min(T, W+128)*2 bytes plus O(B*Hq*T). With a workspace between this and
 * attn_bwd_workspace_bytes the call runs in passes, each over as many (batch, KV head)
 * blocks as the workspace holds (a main and a dQ launch per pass), with the same results. */
size_t attn_bwd_workspace_min_bytes(int B, int T, int Hq, int Hkv, int D, int window);

/*
 * attn_bwd -- gradients of sum(dO * o) for o = attn_fwd(q, k, v):
 *   Delta_i = dO_i . o_i,  P = exp(scale q k^T - lse),  dV = P^T dO,
 *   dS = P * (dO V^T - Delta),  dQ = scale dS K,  dK = scale dS^T Q,
 * with dK, dV summed over the Hq/Hkv query heads of each KV head.
 * Inputs: q, k, v, o, dO (bf16) and lse (fp32) exactly as attn_fwd produced
 * them. Outputs dq (B,T,Hq,D), dk, dv (B,T,Hkv,D) bf16, fully overwritten.
 * workspace: device memory, 256-byte aligned, of ws_bytes >=
 * attn_bwd_workspace_min_bytes(B, T, Hq, Hkv, D, window); attn_bwd_workspace_bytes
 * (or more) runs the call in one pass. Launches: a per-row preparation, then per pass
 * the tensor-core main kernel (dK and dV complete per key tile, the dS^T tiles stored
 * to the workspace) and the tensor-core dQ kernel (dQ = scale dS K from the stored
 * tiles); passes after the first start with a memset of the two work counters. Calls where one (batch, KV head) block's stored dS^T
 * tiles would exceed 2^31 rows, or T_pad * Hq reaches 2^31, return ATTN_ERR_UNSUPPORTED.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                       int T, int Hq, int Hkv, int D, int window, float scale, void* stream);

/* Bytes of workspace attn_block_bwd needs: the same as attn_bwd's (the rotary angles
 * are computed in the kernels, from each row's position). */
size_t attn_block_bwd_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int window);

/*
 * attn_block_bwd -- the backward of the whole attention block of training,
 * prologue included (nanochat Admin & Developer Guide, 3: RMS-norm of q and k
 * without weight, then RoPE at positions t; the softmax backward as in
 * attn_bwd): gradients with respect to the RAW q, k and to v, of sum(dO * o) for
 *   q_hat, k_hat = attn_rope_qknorm(q, k) (pos null),  o = attn_fwd(q_hat, k_hat, v).
 * It computes what attn_bwd followed by attn_rope_qknorm_bwd computes, with the
 * prologue backward done on the way out of the kernels (the dK epilogue of the
 * main kernel and the dQ kernel's epilogue, each on a raw tile it loads by TMA):
 * dq_hat and dk_hat never reach memory.
 *   q (B,T,Hq,D), k (B,T,Hkv,D): the raw inputs of the prologue.
 *   q_hat, k_hat: the prologue's outputs for them (rope_base, eps as given here).
 *   v, o, dO, lse: as for attn_bwd. Outputs dq, dk (raw-input gradients) and dv.
 *   workspace: 256-byte aligned, >= attn_bwd_workspace_min_bytes(...); as for attn_bwd,
 *   less than attn_block_bwd_workspace_bytes(...) runs in passes.
 * Same checks, errors and launches as attn_bwd; rope_base > 1 and eps >= 0.
 */
attn_status_t attn_block_bwd(const void* q, const void* k, const void* q_hat, const void* k_hat, const void* v,
                             const void* o, const void* dO, const float* lse, void* dq, void* dk, void* dv,
                             void* workspace, size_t ws_bytes, int B, int T, int Hq, int Hkv, int D, int window,
                             float scale, float rope_base, float eps, void* stream);

/* Bytes of workspace attn_quantize_fp8 needs for n elements (per-block maxima). */
size_t attn_quantize_fp8_workspace_bytes(long long n);

/*
 * attn_quantize_fp8 -- tensorwise dynamic scaling of a bf16 tensor to float8 e4m3
 * (nanochat Admin & Developer Guide, 5 "Precision: Explicit dtype & FP8": one
 * scale per tensor from its absolute maximum, forward tensors in e4m3):
 *   amax = max |x|,  s = 448 / amax (1 when amax = 0),  x8 = e4m3(x * s)
 * with s and x * s computed in fp32 and the rounding to nearest even, saturating
 * at +-448. Writes the n one-byte codes to x8 and the dequantization factor
 * amax / 448 (x ~ x8 * descale) to *descale, both device memory.
 *   x: n bf16 values, 16-byte aligned, n a multiple of 8; x8: n bytes, 8-byte
 *   aligned; descale: one float, device memory, 4-byte aligned.
 *   workspace: >= attn_quantize_fp8_workspace_bytes(n) bytes of device memory.
 * Two launches (maxima, then codes); nothing else is read or written.
 */
attn_status_t attn_quantize_fp8(const void* x, long long n, void* x8, float* descale, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * attn_fwd_fp8 -- attn_fwd on e4m3 operands (nanochat Admin & Developer Guide, 6
 * "Attention: FA3 with SDPA Fallback": FA3 runs in bf16 or fp8; 5: the tensorwise
 * e4m3 recipe). q8 (B,T,Hq,128), k8, v8 (B,T,Hkv,128): e4m3 codes, one byte per
 * element, BTHD, as attn_quantize_fp8 writes them; descale: three floats in device
 * memory, the dequantization factors of q, k and v in that order. Computes
 *   S = scale * (q8 dq) (k8 dk)^T on the causal window, o = softmax(S) (v8 dv),
 * with the products on the e4m3 tensor cores (fp32 accumulation) and P rounded to
 * e4m3 (scaled by 2^8) for the P V product; the row sums use the unrounded P.
 * o (B,T,Hq,128) bf16, lse (B,Hq,T) fp32 as for attn_fwd. D must be 128
 * (ATTN_ERR_UNSUPPORTED otherwise); other checks as for attn_fwd.
 */
attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* descale, void* o, float* lse,
                           int B, int T, int Hq, int Hkv, int D, int window, float scale, void* stream);

/* Bytes of workspace attn_decode needs: the fp32 split-K partials (B*Hq*chunks*(D+2)*4
 * bytes, chunks = ceil(min(window+1, Tmax) / 128), rounded up to 256) and one 8-byte
 * arrival counter per (sequence, head). Nothing in it needs to be initialised: the
 * counters carry a per-call tag, so stale or garbage contents read as zero. */
size_t attn_decode_workspace_bytes(int B, int Hq, int D, int Tmax, int window);

/*
 * attn_decode -- one new token per sequence against its KV cache
 * (nanochat Admin & Developer Guide, 7 "KV cache"; 6: decode slices the window).
 *   q (B,1,Hq,D) bf16, already through the prologue at position pos[b].
 *   kcache, vcache (B,Tmax,Hkv,D) bf16; pos int32 (B): entries already in
 *   each cache = the new token's position, 0 <= pos[b] < Tmax.
 *   k_new, v_new (B,1,Hkv,D) or both null: when given they are written into
 *   the caches at pos[b] (in place) and attended to; when null the caches must
 *   already hold the new token's entry at pos[b].
 *   The token attends to keys [max(0, pos[b] - window), pos[b]].
 *   o (B,1,Hq,D) bf16; lse (B,Hq) fp32 or null.
 * Any group size Hq/Hkv. A pos[b] out of range leaves NaN in that row's outputs and
 * raises ATTN_ERR_DEVICE in the status word.
 * Memory-bound split-K over 128-key chunks in one launch: every cache byte is read
 * once, and the last chunk of each (sequence, KV head) to finish merges the chunks.
 * Calls that share a workspace must be ordered (one stream): overlapping calls race
 * on it.
 */
attn_status_t attn_decode(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                          const int32_t* pos, void* o, float* lse, int B, int Tmax, int Hq, int Hkv, int D,
                          int window, float scale, void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_prefill -- a chunk of T new tokens per sequence against its KV cache
 * (nanochat Admin & Developer Guide, 6 "Attention: FA3 with SDPA Fallback":
 * chunked / sliding-window inference; 7 "KV cache": (B,T,H,D) caches with int32
 * per-row positions, appended in place).
 *   q (B,T,Hq,D) bf16, already through the prologue at positions pos[b] + t
 *   (attn_rope_qknorm with the same pos does that).
 *   kcache, vcache (B,Tmax,Hkv,D) bf16; pos int32 (B) device: entries already in
 *   each cache, so chunk row t sits at position pos[b] + t; 0 <= pos[b] and
 *   pos[b] + T <= Tmax.
 *   k_new, v_new (B,T,Hkv,D) or both null: when given they are first written into
 *   the caches at rows pos[b] .. pos[b] + T - 1 (in place); when null the caches
 *   must already hold them there.
 *   Chunk row t attends to keys [max(0, p - window), p] of its cache, p = pos[b] + t
 *   (window < 0: [0, p]). Cache rows past pos[b] + T - 1 are never read, so they
 *   may hold anything, NaN included.
 *   o (B,T,Hq,D) bf16, lse (B,Hq,T) fp32 (natural log) or null.
 * All device pointers are caller-owned, 16-byte aligned (pos and lse 4-byte).
 * T <= Tmax, else ATTN_ERR_INVALID_ARG. A sequence whose pos[b] is out of range is
 * neither appended nor computed (its rows of o and lse are left as they were)
 * and raises ATTN_ERR_DEVICE in the status word. One launch: the tensor-core
 * forward reads the chunk's keys from k_new / v_new and copies them into the
 * caches on the way (no cache row at or past pos[b] is read when they are given).
 */
attn_status_t attn_prefill(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                           const int32_t* pos, void* o, float* lse, int B, int T, int Tmax, int Hq, int Hkv, int D,
                           int window, float scale, void* stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device memory.
 * (This entry point has no counterpart on the pages: it is a packaging variant.)
 *
 * Some callers have no way to hand this library a workspace: code that runs
 * inside a framework whose allocator it cannot reach, a serving loop that is
 * not allowed to allocate once it has started, or a host program linked only
 * against this C ABI. This call computes exactly what attn_decode computes
 * (same arguments minus the workspace) but keeps the split-K partials in a
 * fixed scratch array that the library itself holds in device memory.
 *
 *   - Limit: what one call needs, attn_decode_workspace_bytes(B, Hq, D, Tmax,
 *     window) (its partials and arrival counters), must fit in the fixed 4 MiB
 *     scratch (4194304 bytes; e.g. 32 sequences x 16 query heads at window 1024
 *     and D = 128 need 2.4 MB).
 *     Larger calls return ATTN_ERR_INVALID_ARG and enqueue nothing.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *     The scratch is a file-scope __device__ array, so every GPU that loads the
 *     library holds those 4 MiB until the process exits.
 *   - The first call on a device looks the scratch's device address up (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the one scratch, which keeps the last call's
 *     contents. Calls whose kernels overlap on the GPU (different streams, no
 *     ordering between them) race on it and give undefined results; calls on
 *     one stream are safe. No part of it needs to start at zero: every partial
 *     a call reads is written earlier in that same call, and the arrival
 *     counters carry a per-call tag.
 */
attn_status_t attn_decode_noalloc(const void* q, void* kcache, void* vcache, const void* k_new, const void* v_new,
                                  const int32_t* pos, void* o, float* lse, int B, int Tmax, int Hq, int Hkv, int D,
                                  int window, float scale, void* stream);

/*
 * attn_layer_window -- the attention window of one layer of a stack
 * (nanochat Admin & Developer Guide, 3 "Sliding-window attention").
 *   pattern: a NUL-terminated string of 'S' and 'L' tiled over the layers
 *   (nanochat's default is "SSSL"); layer in [0, n_layer).
 * Returns -1 (unbounded: the full context) for an 'L' layer and for the last
 * layer whatever the pattern says; for an 'S' layer short_window when it is > 0,
 * else a quarter of seq_len rounded up to a multiple of 128 (2048 -> 512).
 * Returns -2 for a null or empty pattern, any other character, or sizes out of
 * range. Host only; needs no GPU.
 */
int attn_layer_window(const char* pattern, int layer, int n_layer, int seq_len, int short_window);

/*
 * attn_kv_replicate -- expand a batch-1 prefill cache across N samples
 * (nanochat Admin & Developer Guide, 7 "KV cache" and "Generation flow": the
 * prompt is prefilled once at batch 1, then its cache is copied to every row).
 *   k_src, v_src: (n_layers, 1, Tmax_src, Hkv, D) bf16 device memory.
 *   k_dst, v_dst: (n_layers, N, Tmax, Hkv, D) bf16 device memory.
 * Copies rows [0, rows) of every layer into every sample row; the destination's
 * other rows are left as they were. 0 <= rows <= min(Tmax_src, Tmax); the four
 * buffers must not overlap (ATTN_ERR_INVALID_ARG). The caller sets each
 * sample's position (cache_seqlens) to rows. One launch on `stream`: each vector
 * of the prompt rows is read once and stored to every sample (16-byte vectors when
 * the pointers and the row size allow, else 4 or 2 bytes); a failed launch returns
 * ATTN_ERR_LAUNCH.
 */
attn_status_t attn_kv_replicate(const void* k_src, const void* v_src, void* k_dst, void* v_dst, int n_layers,
                                int rows, int Tmax_src, int N, int Tmax, int Hkv, int D, void* stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: ATTN_OK, ATTN_ERR_TIMEOUT or ATTN_ERR_DEVICE (or
 * ATTN_ERR_LAUNCH if a CUDA error is pending). */
attn_status_t attn_get_status(void* stream);

/*
 * attn_debug_set_wait_limit -- test hook for the failure-detection path.
 * Every wait inside the kernels is bounded: a wait on a pipeline stage (a tile
 * copy, a tensor-core product, another warp's results) that has not completed
 * after the limit gives up, records ATTN_ERR_TIMEOUT in the status word and
 * makes its CTA wind down: every other wait of the CTA falls through, the CTA
 * still waits for the copies and products it issued itself (those waits keep
 * the default limit), frees its tensor memory and exits, leaving the outputs
 * of that call undefined. This call sets the pipeline-wait limit, in
 * nanoseconds, for launches made after it on the current device; 0 restores
 * the default (2 s, also the maximum: a longer limit is ATTN_ERR_INVALID_ARG).
 * A limit of a few nanoseconds makes ordinary waits run out, so a test can
 * check that the status is reported and that the next call with the default
 * limit is correct. It synchronises `stream` first and the device after, and
 * is meant for tests only: the default is the right limit for real work.
 */
attn_status_t attn_debug_set_wait_limit(unsigned long long ns, void* stream);

/* Static description of a status code. */
const char* attn_status_string(attn_status_t status);

/* 1 when the current device is an sm_100 part this library was built for, else 0. */
int attn_device_supported(void);

#ifdef __cplusplus
}
#endif

#endif /* CSWA_ATTN_H */
