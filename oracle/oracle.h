/*
 * oracle.h -- plain, slow, CPU reference for low-bit weight quantization and
 * the quantized linear layer with a low-rank adapter.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this code; only the test-suite, the smoke check and the CPU-baseline leg
 * of the benchmark load it.  It shares no source, header, table or helper with
 * the CUDA library.
 *
 * Sources (web pages; cited by page title and section):
 *  [GB]  GreenBit.AI article on low-bit LLM quantization and training
 *        ("只需单卡RTX 3090，低比特量化训练就能实现LLaMA-3 8B全参微调"),
 *        section 模型量化, step (1): group-wise MinMax quantizer,
 *        INT4 with group size 128 and INT2 with group size 64,
 *        layer-mix and channel-mix layouts.
 *  [BNB] bitsandbytes FSDP-QLoRA guide, section 量化数据的存储 (quant_storage):
 *        4-bit packing with the first code in the high nibble; NF4/FP4;
 *        nested (double) quantization of absmax; compute_dtype (bf16).
 *  [QL]  QLoRA explainer, sections QLoRA技术原理 and 关键技术细节:
 *        4-bit NormalFloat codebook, double quantization of the scale factors
 *        and their offset (about 0.37 bit/param saved), and gradients flowing
 *        through the frozen 4-bit weight into the low-rank adapters.
 *
 * Floating-point contract: every float step is a single IEEE binary32 (or
 * binary64 where stated) operation in round-to-nearest-even; the file is
 * compiled with -ffp-contract=off and without fast-math.
 *
 * Parity pins: every function below is pinned by the not-gpu tests (invariants,
 * closed forms, hand-built vectors, brute force on tiny shapes, finite
 * differences).  See the test files for which pin covers which function.
 *
 * All pointers are host pointers owned by the caller.  Functions returning int
 * return 0 on success and a negative value when a stated precondition fails.
 */
#ifndef LBQ_ORACLE_H
#define LBQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* --- number formats --------------------------------------------------- */
float    oracle_bf16_to_f32(uint16_t b);
uint16_t oracle_f32_to_f16(float x);   /* IEEE round-to-nearest-even */
float    oracle_f16_to_f32(uint16_t h);

/* --- MinMax group quantizer ([GB] 模型量化 step (1)) ------------------ */
/* W: bf16 bits [n, k] row-major; groups of `group` consecutive elements along
 * k.  bits in {2, 4}; group divides k.  Outputs: codes [n, k] (one code per
 * byte, may be NULL), scale and zero as fp16 bits [n, k/group]. */
int  oracle_minmax_quantize(const uint16_t* W, int64_t n, int64_t k, int bits,
                            int group, uint8_t* codes, uint16_t* scale,
                            uint16_t* zero);
/* Pack codes [n, k] into bytes [n, k*bits/8], first code in the high bits. */
int  oracle_pack(const uint8_t* codes, int64_t n, int64_t k, int bits,
                 uint8_t* packed);
int  oracle_unpack(const uint8_t* packed, int64_t n, int64_t k, int bits,
                   uint8_t* codes);
/* W_hat[n, k] = (q - zero) * scale, fp32, exact. */
int  oracle_minmax_dequantize(const uint8_t* packed, const uint16_t* scale,
                              const uint16_t* zero, int64_t n, int64_t k,
                              int bits, int group, float* W_hat);

/* --- 4-bit codebook quantizer with per-64 absmax ([QL], [BNB]) ---------- */
/* codebook: 16 fp32 entries in [-1, 1], in code order, containing a zero
 * (+0 or -0); entries need not be sorted or distinct (the FP4 E2M1 table
 * has both zeros).  codes [n, k] (may be NULL), absmax fp32 [n*k/64]. */
int  oracle_codebook_quantize(const uint16_t* W, int64_t n, int64_t k,
                              const float* codebook, uint8_t* codes,
                              float* absmax);
/* Double quantization of absmax: offset = mean, then per block of 256
 * symmetric int8 with an fp32 scale.  q8 [nb], s2 [ceil(nb/256)], offset [1].
 * Returns -2 when the fp64 sum of absmax is not exact (precondition). */
int  oracle_double_quant(const float* absmax, int64_t nb, int8_t* q8,
                         float* s2, float* offset);
/* absmax' = q8/127 * s2 + offset, each step one fp32 operation. */
int  oracle_double_dequant(const int8_t* q8, const float* s2, float offset,
                           int64_t nb, float* absmax_hat);
/* W_hat = codebook[code] * absmax (absmax is either the raw or the
 * double-dequantized one). */
int  oracle_codebook_dequantize(const uint8_t* packed, const float* absmax,
                                const float* codebook, int64_t n, int64_t k,
                                float* W_hat);

/* --- quantized linear layer with LoRA ([QL] QLoRA技术原理) --------------- */
/* All products in fp64 from bf16 inputs (X, A, B, dY: bf16 bits) and the fp32
 * dequantized weight W_hat [n, k].  rank may be 0 (A, B ignored).
 *   T  = X A^T                  [m, r]
 *   Y  = X W_hat^T + s T B^T    [m, n]
 *   U  = dY B                   [m, r]
 *   dX = dY W_hat + s U A       [m, k]
 *   dA = s U^T X                [r, k]
 *   dB = s dY^T T               [n, r]
 * Each output may be NULL to skip it.  The *_bound outputs receive the
 * per-element magnitude sums used by the parity tolerance:
 *   Ybound[i,j]  = sum_k |x_ik| (|w_jk| + s sum_t |B_jt||A_tk|)
 *   dXbound[i,k] = sum_j |dy_ij| (|w_jk| + s sum_t |B_jt||A_tk|)
 *   dAbound[t,k] = s sum_i |x_ik| sum_j |dy_ij||B_jt|
 *   dBbound[j,t] = s sum_i |dy_ij| sum_k |x_ik||A_tk|                      */
int  oracle_linear_fwd(const uint16_t* X, int64_t m, const float* W_hat,
                       int64_t n, int64_t k, const uint16_t* A,
                       const uint16_t* B, int r, double s, double* Y,
                       double* T, double* Ybound);
int  oracle_linear_bwd(const uint16_t* dY, int64_t m, const float* W_hat,
                       int64_t n, int64_t k, const uint16_t* A,
                       const uint16_t* B, int r, double s, double* dX,
                       double* U, double* dXbound);
int  oracle_lora_grads(const uint16_t* X, const uint16_t* dY, int64_t m,
                       int64_t n, int64_t k, const uint16_t* A,
                       const uint16_t* B, int r, double s, double* dA,
                       double* dB, double* dAbound, double* dBbound);
/* Y (and its bound) at a list of (row, col) pairs only, for sampled parity at
 * full size.  W_hat is given row by row through (packed, scale, zero) of the
 * MinMax format so that the full fp32 matrix need not exist. */
int  oracle_linear_fwd_sampled_minmax(const uint16_t* X, int64_t m,
                                      const uint8_t* packed,
                                      const uint16_t* scale,
                                      const uint16_t* zero, int64_t n,
                                      int64_t k, int bits, int group,
                                      const uint16_t* A, const uint16_t* B,
                                      int r, double s, int64_t npairs,
                                      const int64_t* rows, const int64_t* cols,
                                      double* Y, double* Ybound);

/* dX (and its bound) at a list of (token, feature) pairs only, from the
 * packed MinMax weight (no full fp32 matrix); U = dY B per sampled token. */
int  oracle_linear_bwd_sampled_minmax(const uint16_t* dY, int64_t m,
                                      const uint8_t* packed,
                                      const uint16_t* scale,
                                      const uint16_t* zero, int64_t n,
                                      int64_t k, int bits, int group,
                                      const uint16_t* A, const uint16_t* B,
                                      int r, double s, int64_t npairs,
                                      const int64_t* rows, const int64_t* cols,
                                      double* dX, double* dXbound);

/* --- merging an adapter into the weight ([GB] introduction) ------------ */
/* After fine-tuning, the low-rank module is merged into the full-precision
 * weight.  W_in fp32 [n, k] (the dequantized weight for a merge, a bf16
 * weight widened to fp32 for an unmerge), A bf16 [r, k], B bf16 [n, r],
 * sign +1 (merge) or -1 (unmerge).  Every output element is evaluated in
 * binary32 steps in this order (the pages fix no precision; this order is the
 * definition, so that re-quantizing a merged weight is reproducible):
 *   d = 0;  d = fma(B[i,u], A[u,j], d)  for u = 0 .. r-1
 *   t = s * d
 *   v = W_in[i,j] + t   (merge)   or   W_in[i,j] - t   (unmerge)
 *   W_out[i,j] = bf16 round-to-nearest-even of v
 * r may be 0 (A, B ignored).  W_out: bf16 bits [n, k]. */
int  oracle_lora_merge(const float* W_in, int64_t n, int64_t k,
                       const uint16_t* A, const uint16_t* B, int r, float s,
                       int sign, uint16_t* W_out);

/* Threads used by the loops over rows (OpenMP); 0 keeps the default. */
/* --- channel-mix selection by sensitivity ([GB] 模型量化 (1)) -------------- */
/* score[c] = sum_k m2[k] (e2^2 - e4^2), bound[c] = sum_k m2[k] (e2^2 + e4^2)
 * with m2[k] = mean_t x[t,k]^2 over the calibration activations X [t, k]
 * (bf16) and e4, e2 the errors of the MinMax INT4 g128 / INT2 g64
 * dequantization of W [n, k] (bf16), all in fp64.  k % 128 == 0.
 * bound may be NULL. */
int  oracle_channel_score(const uint16_t* W, int64_t n, int64_t k, const uint16_t* X,
                          int64_t t, double* score, double* bound);
/* perm [n]: the n4 channels of highest score (ties: lower channel first) in
 * ascending order, then the others in ascending order. */
int  oracle_channel_mix_select(const double* score, int64_t n, int64_t n4, int32_t* perm);

void oracle_set_threads(int nthreads);
int  oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
