/*
 * nvfp4kv_oracle.h -- C interface of the CPU oracle for the NVFP4 KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  This header and oracle/nvfp4kv_oracle.cpp are a plain,
 * slow, single-threaded restatement of what the NVFP4 KV-cache path computes.  Only the
 * test suite, the smoke check and the CPU-baseline leg of the benchmark may load it.
 * It shares no code, header, table or constant with the CUDA library, and the CUDA
 * library never calls it.
 *
 * Sources (all web pages on "LongLive-2.0: An NVFP4 Parallel Infrastructure for Long
 * Video Generation"):
 *   [P1]  paper page (paperpeel.com), section 2.2 "NVFP4 Training": 16-element
 *         quantisation blocks, M_FP8 = 448 (largest E4M3 magnitude), M_FP4 = 6 (largest
 *         E2M1 magnitude).
 *   [P1'] same page, section 4.2 "Inference with Multi-Shot Attention Sink": sliding
 *         window of W chunks with a KV cache, permanent global sink, effective key set
 *         K_eff(t) = A_g U A_s U KV[t-W, t) with duplicates removed.
 *   [P1''] same page, section 2.1 "Sequence-Parallel AR Training": a noisy chunk attends
 *         to the preceding clean chunks and to its own tokens.
 *   [N1]  reading note (yingwang.github.io), "The NVFP4 quantization format": E2M1
 *         elements (1 sign, 2 exponent, 1 mantissa bit), an E4M3 scale per 16 elements,
 *         an FP32 scale on top; dequantisation is the product of the three.
 *   [N2]  reading note, "The inference infrastructure": the KV cache is re-quantised at
 *         frame-chunk granularity; storage goes from 4*Tc*H*d to 9/8*Tc*H*d bytes; within a
 *         chunk, K-smoothing is applied to K and adaptive scale selection to V.
 *   [N3]  reading note, "Engineering details of NVFP4 training" (few-step distillation): the
 *         adaptive scale search draws its candidate scale magnitudes from {4, 6}; paper page,
 *         section A.2, names adaptive block-scale selection ("Four Over Six", its reference [12])
 *         as a way to lower NVFP4 quantisation error.
 *
 * Cache format the oracle reads and writes (one tensor, K or V):
 *   codes  uint8 [B][H][T][d/2]   element 2j in the low nibble of byte j, 2j+1 in the high
 *   scales uint8 [B][H][T][d/16]  E4M3 bit patterns, one per 16 consecutive elements of d
 *   gscale fp32  [B][H][C]        one FP32 scale per (batch, head, chunk slot)
 * with T = C * chunk_tokens and chunk slot c holding tokens [c*chunk_tokens, (c+1)*chunk_tokens).
 */
#ifndef NVFP4KV_ORACLE_H
#define NVFP4KV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E2M1 (4-bit) and E4M3 (8-bit) element codecs [N1], [P1]. */
double  oracle_e2m1_decode(uint8_t code);
uint8_t oracle_e2m1_encode(float v);      /* round to nearest, ties to even code, clamp to +-6 */
double  oracle_e4m3_decode(uint8_t code); /* NaN for 0x7F / 0xFF */
uint8_t oracle_e4m3_encode(float v);      /* round to nearest, ties to even code, clamp to +-448 */

/* Element-wise encoders over arrays (out[i] = encode(x[i])), for sweeping conversions. */
void oracle_e2m1_encode_array(const float* x, int64_t n, uint8_t* out);
void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out);

/* Quantise one chunk of one tensor (K or V) for every (b, h).
 * x       : bf16 bit patterns, element (b, t, h, i) at x[(b*L + t)*token_stride + h*d + i]
 * codes   : [B][H][L][d/2], scales: [B][H][L][d/16], gscale: [B][H]
 * Returns 0, or -1 for bad sizes (d not a multiple of 16, non-positive sizes). */
int oracle_quantize_chunk(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                          int64_t token_stride, uint8_t* codes, uint8_t* scales, float* gscale);

/* K-smoothing [N2]: the channel mean of one chunk's keys per (b, h): the exact sum over the chunk's
 * L tokens divided by L, rounded once to fp32 (nearest, ties to even).  mean: [B][H][d].
 * Returns 0, or -1 for bad sizes (L above 2^23 included). */
int oracle_key_mean(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                    int64_t token_stride, float* mean);

/* oracle_quantize_chunk with the pages' two recipe options [N2], [N3]:
 *   mean           : NULL, or [B][H][d]: quantise x - mean (one fp32 subtraction per element)
 *   adaptive_scale : 0, or 1 to choose each block's scale target from {6, 4} by the smaller fp64
 *                    squared error (ties keep 6); g stays A / (448 * 6).
 * With mean NULL and adaptive_scale 0 it is oracle_quantize_chunk.  Returns 0 or -1. */
int oracle_quantize_chunk_ex(const uint16_t* x, int32_t B, int32_t L, int32_t H, int32_t d,
                             int64_t token_stride, const float* mean, int32_t adaptive_scale,
                             uint8_t* codes, uint8_t* scales, float* gscale);

/* Dequantise tokens of a cache tensor into fp64: out[B][H][T][d] = e2m1 * e4m3 * gscale. */
int oracle_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale,
                      int32_t B, int32_t H, int32_t d, int32_t chunk_tokens, int32_t capacity,
                      double* out);

/* Visible chunk slots for a query chunk: {c < n_sink} U {q_chunk-window < c <= q_chunk},
 * duplicates removed, ascending, clipped to [0, capacity).  Writes them to out (room for
 * capacity entries) and returns how many there are, or -1 for bad arguments. */
int oracle_visible_chunks(int32_t q_chunk, int32_t n_sink, int32_t window, int32_t capacity,
                          int32_t* out);

/* The effective chunk set of a multi-shot attention sink (paper page, section 4.2 "Inference with
 * Multi-Shot Attention Sink"; reading note, "Multi-shot attention sinks"): the global sink
 * {c < n_sink}, the current shot's sink {shot_start <= c < shot_start + shot_len} and the sliding
 * window {q_chunk - window < c <= q_chunk}, overlaps counted once, ascending, clipped to
 * [0, capacity); the shot sink must end at or before the query chunk (it is history).
 * shot_len = 0 gives oracle_visible_chunks.  Returns the count or -1. */
int oracle_multishot_chunks(int32_t q_chunk, int32_t n_sink, int32_t window, int32_t shot_start,
                            int32_t shot_len, int32_t capacity, int32_t* out);

/* fp64 attention of selected query rows over the dequantised cache.
 * q       : bf16 bit patterns, element (b, i, h, e) at q[(b*Lq + i)*q_token_stride + h*d + e]
 * rows    : n_rows triples (b, h, i)
 * out     : [n_rows][d] fp64
 * softmax_scale <= 0 selects 1/sqrt(d).  Returns 0 or -1 for bad arguments. */
int oracle_attention_rows(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                          int64_t q_token_stride,
                          const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                          const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                          int32_t chunk_tokens, int32_t capacity,
                          int32_t q_chunk, int32_t n_sink, int32_t window, double softmax_scale,
                          const int32_t* rows, int32_t n_rows, double* out);

/* The same attention over the keys of the listed chunk slots (any order; a slot listed twice counts
 * once; each in [0, capacity); n_slots >= 1).  Returns 0 or -1 for bad arguments. */
int oracle_attention_rows_slots(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                                int64_t q_token_stride,
                                const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                                const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                                int32_t chunk_tokens, int32_t capacity, const int32_t* slots,
                                int32_t n_slots, double softmax_scale, const int32_t* rows,
                                int32_t n_rows, double* out);

/* oracle_attention_rows_slots over smoothed keys: key t of chunk c of (b, h) is x_hat' + mu with
 * mu = k_mean[((b*H + h)*capacity + c)*d ...] (fp32); k_mean NULL gives oracle_attention_rows_slots. */
int oracle_attention_rows_slots_kmean(const uint16_t* q, int32_t B, int32_t Lq, int32_t H, int32_t d,
                                      int64_t q_token_stride,
                                      const uint8_t* k_codes, const uint8_t* k_scales, const float* k_gscale,
                                      const float* k_mean,
                                      const uint8_t* v_codes, const uint8_t* v_scales, const float* v_gscale,
                                      int32_t chunk_tokens, int32_t capacity, const int32_t* slots,
                                      int32_t n_slots, double softmax_scale, const int32_t* rows,
                                      int32_t n_rows, double* out);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4KV_ORACLE_H */
