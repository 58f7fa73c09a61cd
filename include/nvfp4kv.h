/*
 * nvfp4kv.h -- C ABI of libnvfp4kv: an NVFP4 KV cache for chunk-wise autoregressive
 * video-DiT attention on NVIDIA B200 (sm_100a).
 *
 * The method follows the pages on "LongLive-2.0: An NVFP4 Parallel Infrastructure for Long
 * Video Generation":
 *  - paper page (paperpeel.com), section 1 "Introduction" and section 3.2 "Parallel KV
 *    Quantization": the KV cache of the DiT is quantised to NVFP4 and dequantised in
 *    parallel inside the attention kernel;
 *  - reading note (yingwang.github.io), "The inference infrastructure": each new chunk's
 *    K and V are re-quantised at frame-chunk granularity; storage falls from 4*Tc*H*d to
 *    9/8*Tc*H*d bytes;
 *  - reading note, "The NVFP4 quantization format", and paper section 2.2 "NVFP4 Training":
 *    E2M1 elements, one E4M3 scale per 16 elements (largest magnitudes 6 and 448), one FP32
 *    scale on top; dequantisation is the product of the three;
 *  - paper section 4.2 "Inference with Multi-Shot Attention Sink": sliding-window attention
 *    over a KV cache of W chunks plus a permanent global sink and, for multi-shot video, the
 *    current shot's sink, overlaps deduplicated;
 *    section 2.1: a chunk attends to the preceding clean chunks and to its own tokens.
 *
 * Quantisation of one (chunk, head, tensor) with X = chunk_tokens x head_dim bf16 values,
 * every step one fp32 round-to-nearest-even operation:
 *    A = max|x|;  g = A / 2688 (0 if A == 0)                 -- FP32 scale, 2688 = 448 * 6
 *    per token, per 16-element block b along head_dim:
 *      s_b = E4M3_rn_satfinite(max_b|x| / (6 * g))           (0 if max_b|x| == 0 or g == 0)
 *      r   = 1 / (s_b * g);  q_i = E2M1_rn_satfinite(x_i * r) (all 0 if s_b == 0 or r is inf)
 * Dequantisation: x_hat = E2M1(q) * E4M3(s) * g.
 *
 * Recipe options (nvfp4kv_cache.flags).  The reading note, "The inference infrastructure", applies
 * "K-smoothing" to K and "adaptive scale selection" to V within each chunk, and "Engineering
 * details of NVFP4 training" draws the candidate scale magnitudes from {4, 6}; the paper page,
 * section A.2, cites adaptive block-scale selection ("Four Over Six") for lower NVFP4 error.  The
 * pages define neither; this library reads them as:
 *  NVFP4KV_K_SMOOTH: per (chunk, head) the channel mean of the chunk's keys,
 *      mu_e = (sum over t of x[t][e]) / chunk_tokens, computed exactly and rounded once to fp32
 *      (nearest, ties to even; a key with an Inf or NaN bit pattern counts as the finite number
 *      (1 + f / 128) * 2^128 of its fraction bits f),
 *    is stored in k_mean and the chunk is quantised as above from x' = x - mu (one fp32
 *    subtraction per element); the key the cache holds is x_hat' + mu, and attention adds the
 *    per-(query row, chunk) term q . mu to every logit of the chunk's keys.
 *  NVFP4KV_V_ADAPTIVE_SCALE: per block of V both scale targets T = 6 and T = 4 are tried
 *    (s_b = E4M3(max_b|x| / (T * g)), codes as above); the one with the smaller squared error
 *    sum over the block's 16 elements, in order, of (x_i - E2M1(q_i) * E4M3(s_b) * g)^2 (fp64,
 *    each operation rounded once) is kept, ties keep 6.  g is unchanged; dequantisation and
 *    attention read such blocks as any other.
 *
 * CONVENTIONS (all entry points)
 *  - Every pointer named "device" is CUDA device memory owned by the caller; the library
 *    never allocates or frees device memory.  It keeps no state between calls other than
 *    per-process caches (driver entry points, per-shape launch plans and occupancy answers)
 *    and the fixed 64 KiB scratch array of nvfp4_kv_quantize_static_scratch.
 *  - Calls are asynchronous on the given CUDA stream (a cudaStream_t passed as void*, NULL
 *    means the legacy default stream).  The return value reports host-side argument checks
 *    and launch errors only.  Errors found on the device (a bounded wait that ran out) are
 *    OR-ed into the cache's device status word; read it with nvfp4kv_read_status().
 *  - Inputs must be finite.  Non-finite input is a precondition violation, not detected.
 *  - Supported: head_dim == 128, chunk_tokens even, sm_100a device.
 */
#ifndef NVFP4KV_H
#define NVFP4KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4KV_OK = 0,
  NVFP4KV_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, bad slot */
  NVFP4KV_ERR_UNSUPPORTED = 2,    /* head_dim != 128, odd chunk_tokens, non-sm_100 device */
  NVFP4KV_ERR_CUDA = 3,           /* a CUDA runtime or driver call failed */
  NVFP4KV_ERR_DEVICE_TIMEOUT = 4, /* status bit: a kernel's bounded wait ran out */
  NVFP4KV_ERR_WORKSPACE = 5       /* workspace pointer null or smaller than required */
} nvfp4kv_status;

typedef enum { NVFP4KV_OUT_F32 = 0, NVFP4KV_OUT_BF16 = 1 } nvfp4kv_out_dtype;

/* One layer's NVFP4 KV cache.  T = capacity_chunks * chunk_tokens; chunk slot c holds
 * tokens [c*chunk_tokens, (c+1)*chunk_tokens).  All arrays are device memory:
 *   k_codes, v_codes   uint8 [batch][heads][T][head_dim/2]   E2M1 pairs, element 2j in the
 *                                                           low nibble of byte j
 *   k_scales, v_scales uint8 [batch][heads][T][head_dim/16]  E4M3 block scales
 *   k_gscale, v_gscale fp32  [batch][heads][capacity_chunks] FP32 scale per chunk
 *   status             uint32, one word; zero it once before first use
 *   k_mean             fp32  [batch][heads][capacity_chunks][head_dim] (NVFP4KV_K_SMOOTH only)
 * Every array must start on a 16-byte boundary.  flags with bits other than the two options,
 * or NVFP4KV_K_SMOOTH without k_mean, is NVFP4KV_ERR_INVALID_ARG for every call, and
 * NVFP4KV_K_SMOOTH with chunk_tokens > 2^23 is NVFP4KV_ERR_UNSUPPORTED for every call; one cache
 * keeps its flags for its whole life (its slots are read as they were written). */
typedef struct {
  int32_t batch;
  int32_t heads;
  int32_t head_dim;
  int32_t chunk_tokens;
  int32_t capacity_chunks;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint8_t* k_scales;
  uint8_t* v_scales;
  float* k_gscale;
  float* v_gscale;
  uint32_t* status;
  uint32_t flags;  /* 0, or recipe options: NVFP4KV_K_SMOOTH | NVFP4KV_V_ADAPTIVE_SCALE */
  float* k_mean;   /* with NVFP4KV_K_SMOOTH: fp32 [batch][heads][capacity_chunks][head_dim], the
                      channel mean of each chunk slot's keys; else unused (may be NULL) */
} nvfp4kv_cache;

/* Recipe option bits of nvfp4kv_cache.flags (see the file header). */
enum { NVFP4KV_K_SMOOTH = 1u, NVFP4KV_V_ADAPTIVE_SCALE = 2u };

/* Bytes of each cache array for the given shape (per tensor, K or V): codes, scales and
 * FP32 scales.  Any output pointer may be NULL.  Returns NVFP4KV_OK or
 * NVFP4KV_ERR_INVALID_ARG for non-positive sizes or head_dim not a multiple of 16. */
int nvfp4kv_cache_sizes(int32_t batch, int32_t heads, int32_t head_dim, int32_t chunk_tokens,
                        int32_t capacity_chunks, size_t* codes_bytes, size_t* scales_bytes,
                        size_t* gscale_bytes);

/* Workspace bytes nvfp4_kv_quantize and the attention calls need for this cache and a query
 * chunk of q_tokens tokens (the maximum over the calls; 0 is never returned).  The attention
 * part holds the partial results of work items split between CTAs: two slots of about 130 KB
 * per SM of the CURRENT device (148 SMs are assumed when no device can be queried), so call it
 * with the device that will run the attention current.  Returns 0 for an invalid cache
 * description. */
size_t nvfp4kv_workspace_bytes(const nvfp4kv_cache* cache, int32_t q_tokens);

/* Quantise a new frame chunk's K and V and write it into chunk slot `chunk_slot`: the
 * re-quantisation of each new frame chunk's K and V into the NVFP4 cache (reading note,
 * "The inference infrastructure"), in the three-level format of the reading note, "The NVFP4
 * quantization format", and paper page section 2.2 (constants 16, 448, 6).
 *   k_bf16, v_bf16  device bf16, element (b, t, h, e) at [(b*chunk_tokens + t)*token_stride +
 *                   h*head_dim + e]; 16-byte aligned; token_stride >= heads*head_dim and a
 *                   multiple of 8
 *   workspace       device scratch of at least nvfp4kv_workspace_bytes() bytes, 16-byte
 *                   aligned; its contents on entry do not matter
 * Writes codes, scales and the FP32 scales of slot `chunk_slot` for every (b, h) (and, with
 * NVFP4KV_K_SMOOTH, the slot's channel means in k_mean); nothing else in the cache is touched.
 * Bit-for-bit deterministic, and the same bits whichever kernel path runs
 * (nvfp4kv_quantize_launches tells which; a cache with recipe options always takes the
 * two-pass path, after a channel-mean kernel when K is smoothed).
 * Errors: NVFP4KV_ERR_INVALID_ARG (null, misaligned, slot out of range, bad stride),
 * NVFP4KV_ERR_UNSUPPORTED, NVFP4KV_ERR_WORKSPACE, NVFP4KV_ERR_CUDA (launch failed); a device
 * wait that ran out sets the status bit of NVFP4KV_ERR_DEVICE_TIMEOUT. */
int nvfp4_kv_quantize(const nvfp4kv_cache* cache, int32_t chunk_slot, const void* k_bf16,
                      const void* v_bf16, int64_t token_stride, void* workspace,
                      size_t workspace_bytes, void* cuda_stream);

/* nvfp4_kv_quantize for the same new chunk slot of several layers' caches in one launch (the
 * per-layer K and V of one generated frame chunk, as the reading note's "The inference
 * infrastructure" re-quantises them).  Results are bit-identical to one nvfp4_kv_quantize call
 * per layer.  The input crosses HBM once: a CTA reduces the maximum of one 128-token part of a
 * (layer, tensor, b, h) slice, and encodes an earlier part once that part's slice is complete,
 * re-reading rows that are still in L2.
 *   caches         host array of n_layers cache descriptors, 1 <= n_layers <= 64, all with the
 *                  same batch, heads, chunk_tokens and capacity
 *   k_bf16, v_bf16 host arrays of n_layers device pointers, each laid out as for
 *                  nvfp4_kv_quantize with the common token_stride
 *   workspace      device scratch of at least nvfp4kv_quantize_layers_workspace_bytes() bytes;
 *                  the call zeroes the counters it keeps there (a memset on the stream), so its
 *                  contents on entry do not matter
 * A device wait that runs out sets the timeout bit in caches[0]'s status word.  Errors as for
 * nvfp4_kv_quantize; NVFP4KV_ERR_INVALID_ARG also for caches of different shapes and
 * NVFP4KV_ERR_UNSUPPORTED for more than 64 layers, more than 2^31 parts, or caches with recipe
 * options (quantise those one layer at a time with nvfp4_kv_quantize). */
int nvfp4_kv_quantize_layers(const nvfp4kv_cache* caches, int32_t n_layers, int32_t chunk_slot,
                             const void* const* k_bf16, const void* const* v_bf16, int64_t token_stride,
                             void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Workspace bytes of nvfp4_kv_quantize_layers for n_layers caches shaped like caches[0]
 * (0 for an invalid description). */
size_t nvfp4kv_quantize_layers_workspace_bytes(const nvfp4kv_cache* caches, int32_t n_layers);

/* nvfp4_kv_quantize without a workspace, for callers that cannot allocate device memory
 * (a pre-planned arena sized before this library was linked, a host framework that owns
 * every device allocation, a real-time loop that must not allocate).  The pages have no
 * counterpart: this is a library convenience, not part of the method.
 * Same arguments, results and errors as nvfp4_kv_quantize, except that the amax partials
 * live in a fixed 64 KiB device array inside the library, which every GPU that loads the
 * library keeps until the process exits.  It calls no cudaMalloc or cudaFree.
 *  - Caches needing more partials than fit (2 * batch * heads * ceil(chunk_tokens / 128) * 4
 *    bytes) are rejected with NVFP4KV_ERR_WORKSPACE before anything is launched; use
 *    nvfp4_kv_quantize for them.
 *  - The first call on each device looks up the array's device address (with that device
 *    current), which may load the library's GPU code: make that first call before any
 *    stream capture.  The address is kept until the process exits; resetting a device
 *    (cudaDeviceReset) while the library is loaded is not supported by this entry point.
 *  - All calls share the one array and every call overwrites what it reads, so nothing needs
 *    clearing between calls; calls that may overlap on the GPU (unordered streams) race. */
int nvfp4_kv_quantize_static_scratch(const nvfp4kv_cache* cache, int32_t chunk_slot,
                                     const void* k_bf16, const void* v_bf16, int64_t token_stride,
                                     void* cuda_stream);

/* Attention of a chunk of bf16 queries over the NVFP4 cache, dequantised inside the kernel
 * (paper page, section 1 and section 3.2 "Parallel KV Quantization"), with the sliding window
 * and permanent sink of paper page section 4.2 and the chunk's own tokens (section 2.1).  The
 * query chunk `q_chunk` attends to the keys of the visible chunk slots
 *     V = { c < n_sink_chunks } U { q_chunk - window_chunks < c <= q_chunk },
 * each slot once (its own chunk included, so it must have been quantised first):
 *     out_i = sum_j softmax_j(scale * q_i . k_hat_j) v_hat_j    over the keys j of V.
 *   q_bf16     device bf16, element (b, i, h, e) at [(b*q_tokens + i)*q_token_stride +
 *              h*head_dim + e]; 16-byte aligned; q_token_stride >= heads*head_dim and a
 *              multiple of 8
 *   out        device [batch][q_tokens][heads][head_dim], fp32 or bf16 (out_dtype),
 *              contiguous, 16-byte aligned
 *   softmax_scale <= 0 selects 1/sqrt(head_dim)
 *   workspace  device scratch of at least nvfp4kv_workspace_bytes(cache, q_tokens) bytes (with
 *              the same device current); contents on entry do not matter
 * With NVFP4KV_K_SMOOTH, k_hat_j is x_hat'_j + mu(chunk of j): the kernel adds scale * q_i . mu
 * per (query row, chunk) to the logits; such caches need chunk_tokens >= 128 (else
 * NVFP4KV_ERR_UNSUPPORTED), so that a 128-key tile spans at most two chunks.
 * One launch of a persistent kernel (one CTA per SM), followed by a small merge kernel when some
 * work item's KV tiles were split between CTAs.  Chunk slots outside V are never read.  Errors as
 * for nvfp4_kv_quantize; window_chunks < 1, n_sink_chunks < 0 or q_chunk outside
 * [0, capacity) give NVFP4KV_ERR_INVALID_ARG. */
int nvfp4_kv_attention(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                       int64_t q_token_stride, int32_t q_chunk, int32_t n_sink_chunks,
                       int32_t window_chunks, float softmax_scale, void* out, int32_t out_dtype,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Attention over an explicit set of visible chunk slots: the multi-shot sink of the paper page,
 * section 4.2 "Inference with Multi-Shot Attention Sink", and the reading note, "Multi-shot
 * attention sinks", where besides the global sink each shot keeps its own sink chunks.  The caller
 * lists the slots (global sink, shot sinks, local window, in any order; repeats are counted once):
 *     out_i = sum_j softmax_j(scale * q_i . k_hat_j) v_hat_j    over the keys j of the listed slots.
 *   slots    host int32[n_slots], each in [0, capacity); n_slots >= 1
 * The slots, sorted, may form at most 4 runs of consecutive slots (more gives
 * NVFP4KV_ERR_UNSUPPORTED before anything is launched).  Other arguments, results and errors as
 * for nvfp4_kv_attention, which is this call with the slots V(q_chunk) above. */
int nvfp4_kv_attention_slots(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                             int64_t q_token_stride, const int32_t* slots, int32_t n_slots,
                             float softmax_scale, void* out, int32_t out_dtype, void* workspace,
                             size_t workspace_bytes, void* cuda_stream);

/* Multi-shot attention sink with the effective key set built inside the library: the paper
 * page, section 4.2 "Inference with Multi-Shot Attention Sink", and the reading note,
 * "Multi-shot attention sinks": besides the permanent global sink each shot keeps the chunks
 * at its start as its own sink, and the query chunk attends to
 *     K_eff = { c < n_sink_chunks }                                     global sink
 *           U { shot_start <= c < shot_start + shot_len }               current shot's sink
 *           U { q_chunk - window_chunks < c <= q_chunk }                sliding window
 * each slot once.  The shot's sink is history: shot_start >= 0, shot_len >= 0 and
 * shot_start + shot_len <= q_chunk + 1, else NVFP4KV_ERR_INVALID_ARG (shot_len == 0 gives
 * nvfp4_kv_attention).  Other arguments, results and errors as for nvfp4_kv_attention; the set
 * may form at most 4 runs of consecutive slots (it forms at most 3). */
int nvfp4_kv_attention_multishot(const nvfp4kv_cache* cache, const void* q_bf16, int32_t q_tokens,
                                 int64_t q_token_stride, int32_t q_chunk, int32_t n_sink_chunks,
                                 int32_t window_chunks, int32_t shot_start, int32_t shot_len,
                                 float softmax_scale, void* out, int32_t out_dtype, void* workspace,
                                 size_t workspace_bytes, void* cuda_stream);

/* Dequantise chunk slots [first_slot, first_slot + n_slots) of K (which == 0) or V
 * (which == 1) into device fp32 out[batch][heads][n_slots*chunk_tokens][head_dim]: the
 * pages' dequantisation step on its own, for tests and diagnostics.  Each value is the
 * exact E2M1 * E4M3 product times the FP32 scale, rounded once to fp32; for K of a cache with
 * NVFP4KV_K_SMOOTH the chunk's channel mean is then added (a second fp32 rounding). */
int nvfp4_kv_dequantize(const nvfp4kv_cache* cache, int32_t which, int32_t first_slot,
                        int32_t n_slots, float* out, void* cuda_stream);

/* Diagnostic probe of the device conversions the quantiser uses: for each of the n fp32
 * values x (device), write the E2M1 code (low nibble; round to nearest even, saturate to
 * +-6) to e2m1_codes and the E4M3 code (round to nearest even, saturate to +-448) to
 * e4m3_codes (both device uint8[n]).  Used to compare the hardware conversions with the
 * format definition over whole ranges of inputs. */
int nvfp4kv_debug_encode(const float* x, int64_t n, uint8_t* e2m1_codes, uint8_t* e4m3_codes,
                         void* cuda_stream);

/* The work split the attention calls use for q_tokens queries over kv_tiles visible KV tiles of
 * 128 keys on n_sms SMs (n_sms <= 0: the current device's count; any n_sms > 0 needs no GPU).  A
 * work item is two query tiles of 128 rows of one (batch, head) (the last item of a head holds one
 * tile when their number is odd) over all kv_tiles KV tiles; the (item, KV tile) units are dealt to
 * out[0] persistent CTAs as contiguous ranges of equal weighted cost, so a CTA's range is a list of
 * segments (parts of consecutive items).  A library diagnostic with no counterpart in the pages.
 *   cta < 0:  out[0] = CTAs, out[1] = kernels per call (2 when some item is split between CTAs and
 *             the merge kernel runs, else 1)
 *   cta >= 0: out[0] = CTAs, out[1] = segments of that CTA; for 0 <= seg < out[1] also
 *             out[2] = batch * heads + head index, out[3] = first query row, out[4] = query tiles
 *             (1 or 2, clipped to q_tokens by the kernel), [out[5], out[6]) = the KV tiles of the
 *             item the segment covers, out[7] = its partial-result slot in the workspace, or -1
 *             when it covers the whole item and writes the output itself
 * Errors: NVFP4KV_ERR_INVALID_ARG (bad cache, q_tokens or kv_tiles <= 0, null out, cta >= out[0],
 * seg >= out[1]), NVFP4KV_ERR_UNSUPPORTED (too many units), NVFP4KV_ERR_CUDA (n_sms <= 0 without
 * a device). */
int nvfp4kv_attention_plan(const nvfp4kv_cache* cache, int32_t q_tokens, int32_t kv_tiles, int32_t n_sms,
                           int32_t cta, int32_t seg, int32_t* out);

/* Kernels that nvfp4_kv_quantize (and its static-scratch variant) launch per call for this cache
 * shape on the current device: 1 when every (batch, head, tensor) gets one thread-block cluster
 * in a single wave (single pass: the input crosses HBM once), 2 otherwise (an amax pass and an
 * encode pass).  Both paths write the same bits.  A library diagnostic with no counterpart in
 * the pages; a negative result is minus an nvfp4kv_status code (invalid cache, no sm_100 device). */
int nvfp4kv_quantize_launches(const nvfp4kv_cache* cache);

/* Fault injection for tests of the failure path, no counterpart in the pages: launches a one-warp
 * kernel whose bounded wait is made to run out (nothing ever arrives at its barrier).  After the
 * kernels' wait limit (about 1 s) it ORs 1 << NVFP4KV_ERR_DEVICE_TIMEOUT into the cache's status
 * word and returns; the CUDA context stays usable.  No GPU fault, trap or hang is involved.
 * Errors: NVFP4KV_ERR_INVALID_ARG (bad cache), NVFP4KV_ERR_UNSUPPORTED, NVFP4KV_ERR_CUDA. */
int nvfp4kv_debug_wait_timeout(const nvfp4kv_cache* cache, void* cuda_stream);

/* Wait for `cuda_stream`, then read the cache's device status word into *out and clear it.
 * *out == 0 means no device-side error since the last read; otherwise it holds OR-ed
 * nvfp4kv_status bits (1 << NVFP4KV_ERR_DEVICE_TIMEOUT for a bounded wait that ran out). */
int nvfp4kv_read_status(const nvfp4kv_cache* cache, void* cuda_stream, uint32_t* out);

/* Static description of a status code.  Never NULL. */
const char* nvfp4kv_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4KV_H */
