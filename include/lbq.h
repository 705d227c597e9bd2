/*
 * lbq.h -- C ABI of the low-bit quantized linear layer library for B200
 * (sm_100a).  All entry points are `extern "C"`, take plain pointers and sizes,
 * and launch asynchronously on the caller's CUDA stream.
 *
 * Sources (web pages, cited by title and section):
 *  - GreenBit.AI article "只需单卡RTX 3090，低比特量化训练就能实现LLaMA-3 8B全参微调",
 *    section 模型量化, step (1): group-wise MinMax quantizer; INT4 with group
 *    size 128 and INT2 with group size 64; layer-mix and channel-mix layouts.
 *    Its introduction: after QLoRA fine-tuning the low-rank module is merged
 *    into the full-precision model (lbq_merge_lora, lbq_unmerge_lora).
 *  - bitsandbytes FSDP-QLoRA guide, section 量化数据的存储 (quant_storage):
 *    two 4-bit codes per byte with the first code in the high nibble; NF4/FP4
 *    codebooks; nested quantization of absmax; weights are dequantized to the
 *    compute dtype (bf16) inside the kernels.
 *  - QLoRA explainer, sections QLoRA技术原理 / 关键技术细节 / 结论: 4-bit
 *    NormalFloat codebook, double quantization of the scale factors and their
 *    offset (about 0.37 bit per parameter saved), and backpropagation through
 *    the frozen 4-bit weight into the low-rank adapters.
 *
 * Conventions
 *  - W is [n out, k in] row-major; quantization groups run along k.
 *  - bf16 and fp16 data are passed as their 16-bit patterns (uint16_t / void*).
 *  - Every pointer in lbq_qweight and every data pointer argument is DEVICE
 *    memory owned by the caller.  The library allocates nothing; it never
 *    frees, retains or reallocates caller memory.
 *  - Device pointers must be 16-byte aligned (LBQ_EALIGN otherwise); sizes
 *    must satisfy the per-function constraints (LBQ_EINVAL otherwise).
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call launches nothing.  Launch failures are reported as
 *    LBQ_ECUDA.  Kernels that wait on a device-side condition give up after a
 *    bounded number of polls and record LBQ_ETIMEOUT in the device status word,
 *    read with lbq_device_status().  Nothing aborts the process.
 *  - Results are deterministic: the same inputs give the same bits.
 */
#ifndef LBQ_H
#define LBQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Compatible with cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* lbq_stream_t;

typedef enum {
    LBQ_OK = 0,
    LBQ_EINVAL = 1,        /* bad shape, bit width, group, scheme or NULL pointer */
    LBQ_EALIGN = 2,        /* a device pointer is not 16-byte aligned */
    LBQ_EUNSUPPORTED = 3,  /* valid request that this build does not implement */
    LBQ_ECUDA = 4,         /* a CUDA runtime call or launch failed */
    LBQ_ETIMEOUT = 5,      /* a device-side wait gave up (see lbq_device_status) */
    LBQ_EWORKSPACE = 6     /* workspace missing or smaller than the query said */
} lbq_status;

typedef enum {
    LBQ_MINMAX_ASYM = 0,   /* group-wise asymmetric MinMax, INT4 g128 / INT2 g64 */
    LBQ_CODEBOOK4 = 1      /* 4-bit codebook with per-64 absmax (NF4-style) */
} lbq_scheme;

/*
 * A quantized weight.  All pointers are caller-owned DEVICE memory.
 *
 * LBQ_MINMAX_ASYM (GreenBit article, 模型量化 (1)):
 *   bits in {4, 2}, group in {128 (bits 4), 64 (bits 2)}, k % group == 0,
 *   k % 64 == 0.  For each row and group of `group` consecutive k:
 *     scale = fp16(fp32(max - min) / Q), Q = 2^bits - 1 (1.0 if that is 0),
 *     zero  = fp16(rint(-min / scale)),
 *     code  = clamp(rint(w / scale) + zero, 0, Q)            (rint: half-even)
 *   packed [n, k*bits/8] u8: codes in order, first code in the high bits.
 *   scale, zero [n, k/group] fp16 bit patterns.
 *   Dequantized value: (code - zero) * scale.
 *
 * LBQ_CODEBOOK4 (QLoRA explainer, 关键技术细节 1; bitsandbytes guide, nf4/fp4):
 *   bits 4, group 64 (blocks of 64 consecutive elements of the row-major W),
 *   k % 64 == 0.  codebook: 16 fp32 values in code order (device memory, read
 *   only), all in [-1, 1], at least one of them a zero; they need not be
 *   sorted or distinct (an NF4-style table is sorted; the FP4 E2M1 table,
 *   bitsandbytes guide "nf4与fp4", holds +0 at code 0 and -0 at code 8), but
 *   distinct values must be at least 2^-20 apart (otherwise lbq_quantize
 *   sets LBQ_STATUS_BAD_TABLE in the device status word).
 *   absmax [n*k/64] fp32 = max |w| per block; code = index of the entry
 *   nearest to fp32(w / absmax) in fp32, the lower index on a tie (so of two
 *   equal entries the lower code is the one produced; a zero goes to the
 *   lowest zero code).  packed [n, k/2] u8 as above.
 *   Dequantized value: codebook[code] * absmax.
 *   With double_quant != 0 (QLoRA explainer, 结论; bitsandbytes guide, nested
 *   absmax): offset = fp32(fp64 sum of absmax / (n*k/64)); per block of 256
 *   absmax values s2 = max |absmax - offset| and
 *   q8 = clamp(rint(fp32(fp32((absmax - offset) / s2) * 127)), -127, 127);
 *   absmax' = fp32(fp32(fp32(q8 / 127) * s2) + offset) replaces absmax in the
 *   dequantized value.  absmax_q8 [n*k/64] i8, absmax_s2 [ceil(n*k/64/256)]
 *   fp32, absmax_offset [1] fp32.  absmax is still required: lbq_quantize
 *   writes the first-level values there.  The offset is reproducible bit for
 *   bit whenever the fp64 sum of the absmax values is exact, which holds when
 *   they span less than 2^(45 - log2(n*k/64)) in magnitude.
 */
typedef struct {
    int32_t n, k;
    int32_t bits, group;
    int32_t scheme;         /* lbq_scheme */
    int32_t double_quant;   /* CODEBOOK4 only */
    uint8_t* packed;
    uint16_t* scale;        /* MINMAX */
    uint16_t* zero;         /* MINMAX */
    float* absmax;          /* CODEBOOK4 */
    int8_t* absmax_q8;      /* CODEBOOK4 + double_quant */
    float* absmax_s2;       /* CODEBOOK4 + double_quant */
    float* absmax_offset;   /* CODEBOOK4 + double_quant */
    const float* codebook;  /* CODEBOOK4 */
} lbq_qweight;

/*
 * Channel-mix layout (GreenBit article, 模型量化 (1)): inside one matrix some
 * output channels are INT4 g128 and the rest INT2 g64.  The rows are stored as
 * two contiguous MinMax matrices, `hi` (INT4) then `lo` (INT2), with the same
 * k; perm[i] (0 <= i < hi.n + lo.n) is the original output channel of stored
 * row i (rows of `hi` first).  Y is produced in the original channel order.
 * hi.n and lo.n may be any sizes >= 1.
 */
typedef struct {
    lbq_qweight hi;
    lbq_qweight lo;
    const int32_t* perm;    /* device, hi.n + lo.n entries, a permutation */
} lbq_qweight_mix;

/* Human-readable name of a status code (static string). */
const char* lbq_status_string(lbq_status s);

/*
 * Quantize and pack W (bf16 [q->n, q->k], device) into q.  Fills packed and
 * scale/zero (MINMAX) or absmax (+ q8, s2, offset with double_quant)
 * (CODEBOOK4).  CODEBOOK4 with double_quant needs a workspace of
 * lbq_quantize_workspace_size(q) bytes (device, any contents); every other
 * case needs none (workspace may be NULL).
 */
size_t lbq_quantize_workspace_size(const lbq_qweight* q);
lbq_status lbq_quantize(const void* W_bf16, lbq_qweight* q, void* workspace,
                        size_t workspace_bytes, lbq_stream_t stream);

/*
 * Dequantize q into W_f32 [q->n, q->k] fp32 (device).  MINMAX values are exact
 * ((code - zero) * scale is one fp32 product); CODEBOOK4 values are
 * fp32(codebook[code] * absmax) with absmax' when double_quant is set.
 */
lbq_status lbq_dequantize(const lbq_qweight* q, float* W_f32,
                          lbq_stream_t stream);

/*
 * Merge the low-rank adapter into the weight (GreenBit article,
 * introduction: after QLoRA fine-tuning the LoRA module is merged into the
 * full-precision model):
 *   W_out[i, j] = bf16( W_hat[i, j] + s * sum_u B[i, u] A[u, j] )
 * W_hat is q dequantized exactly as lbq_dequantize does; A bf16 [rank, k] and
 * B bf16 [q->n, rank] row-major; W_out bf16 [q->n, q->k] row-major.  All
 * device pointers, caller-owned, 16-byte aligned.  Each element is evaluated
 * in binary32 in this order: d = 0, then d = fma(B[i,u], A[u,j], d) for
 * u = 0 .. rank-1; t = s * d; v = W_hat + t; W_out = v rounded to bf16
 * (nearest, ties to even).  The order is part of the contract: the merged
 * weight, and lbq_quantize of it (re-quantizing the merged model), are
 * reproducible bit for bit.  rank == 0 (A, B may be NULL) writes bf16(W_hat).
 * 0 <= rank <= 64.  Returns LBQ_EINVAL / LBQ_EALIGN on bad arguments before
 * any launch.
 */
lbq_status lbq_merge_lora(const lbq_qweight* q, const void* A, const void* B,
                          int rank, float s, void* W_out, lbq_stream_t stream);

/*
 * Remove a merged adapter: W_out = bf16(W - s * B A) for a bf16 weight W
 * [n, k] (device, row-major), with the same binary32 order as lbq_merge_lora
 * and v = W - t.  k must be a multiple of 8; W_out may be W (in place).
 */
lbq_status lbq_unmerge_lora(const void* W, int n, int k, const void* A,
                            const void* B, int rank, float s, void* W_out,
                            lbq_stream_t stream);

/*
 * Forward of the quantized linear layer with a low-rank adapter (QLoRA
 * explainer, QLoRA技术原理):
 *   T = X A^T  [m, rank]                         (fp32, written to T_save)
 *   Y = X W^T + s T B^T  [m, n]                  (fp32)
 * X bf16 [m, k], A bf16 [rank, k], B bf16 [n, rank], all row-major device.
 * rank == 0 (A, B, T_save may be NULL) is the plain dequantize-GEMM.
 * 1 <= rank <= 64 needs T_save.  m >= 1.  The weight is dequantized to bf16
 * (the compute dtype) inside the kernel and products accumulate in fp32.
 * workspace: lbq_linear_fwd_workspace_size(m, q, rank) bytes of device memory,
 * zero-filled before the first call that uses it; NULL is accepted when that
 * size is 0.  It holds split-K partial sums and per-tile arrival counters.
 * For m > 16 the size includes the partial sums of an optional split of the
 * GEMM's last wave of tiles: a smaller workspace is accepted as long as it
 * holds what the call requires (the last wave then runs unsplit, with the
 * same results within the stated bound);
 * every call leaves the counters at zero again, so one zero-fill at
 * allocation serves any number of later calls of any shape.  After a call
 * whose kernels timed out (LBQ_ETIMEOUT from lbq_device_status), zero it
 * again.  Calls that may run at the same time need separate workspaces.
 *
 * Overlap with the previous kernel: for m <= 16 the kernel is launched with
 * programmatic stream serialisation and may start streaming the packed
 * weight and its scales/zeros while the kernel before it on `stream` is
 * still running (X, the workspace, Y and T_save are touched only after that
 * kernel has finished).  When the previous library call on `stream` was
 * lbq_quantize, the forward waits instead.  A caller's own kernel that
 * writes the packed weight or its constants must not directly precede the
 * forward on the same stream (record an event or launch through another
 * stream in between).
 */
size_t lbq_linear_fwd_workspace_size(int m, const lbq_qweight* q, int rank);

/*
 * The decode plan that the forward uses for 1 <= m <= 16 (host only: no
 * device work, no GPU needed) for one launch over `count` weights
 * (1 <= count <= 8; qs[i] are host pointers; only n, k, bits, group,
 * scheme and double_quant are read).  The work of weight i is its
 * (128-row tile, 64-column k-block) units, row tiles x k/64 of them in
 * tile-major order, cut into equal contiguous CTA shares; every CTA of the
 * launch gets about the same bytes and the launch is one wave of two CTAs per
 * SM.  On success plan[0..7] = CTAs, ring stages, stage bytes, dynamic shared
 * memory per CTA, workspace bytes, the SM count the plan was made for (`sms`;
 * when sms <= 0, the current device's, or 148 without one), the bytes of the
 * largest activation box of a stage and the row stride of the per-warp
 * constant buffers; when per_problem is not
 * NULL, per_problem[4i .. 4i+3] = k-blocks per CTA (share), CTAs, first CTA
 * and row tiles of weight i.  Returns LBQ_EINVAL for m outside 1..16, count
 * outside 1..8, a NULL plan or qs, or an invalid descriptor.
 */
lbq_status lbq_gemv_plan(int m, const lbq_qweight* const* qs, int count, int sms,
                         int64_t* plan, int64_t* per_problem);
lbq_status lbq_linear_fwd(const void* X, int m, const lbq_qweight* q,
                          const void* A, const void* B, int rank, float s,
                          float* Y, float* T_save, void* workspace,
                          size_t workspace_bytes, lbq_stream_t stream);

/*
 * lbq_linear_fwd_noalloc -- the same forward as lbq_linear_fwd for callers
 * that cannot allocate device memory: code whose device memory is all handed
 * out up front by another runtime's pool, real-time or embedded loops that
 * must not allocate after start-up, and callers for whom a cudaMalloc (which
 * can synchronize the device) is not allowed at the point of the call.  It
 * takes no workspace: the split-K scratch of both forward paths (the decode
 * GEMV for m <= 16 and the tensor-core GEMM when it splits K) lives in a fixed
 * array of 8 MiB (8388608 bytes) that the library declares once per device
 * and every device that loads the library keeps until the process exits.
 * (The source pages have no counterpart of this entry point.)
 *
 * Arguments, layouts, results and errors are those of lbq_linear_fwd, plus:
 *  - LBQ_EWORKSPACE when the scratch this call requires is larger than the
 *    8 MiB array; nothing is launched then (for m <= 16 it is
 *    lbq_linear_fwd_workspace_size, which tells in advance; for m > 16 that
 *    query may report more, for an optional split of the last wave of tiles
 *    that the call then leaves out when it does not fit).
 *  - Every call looks up the array's device address with the current device
 *    current; the first call on a device may load the library's module, so
 *    make it before any stream capture.
 *  - All calls share the one array: calls that can run at the same time on
 *    the GPU (different streams, overlapping graphs) race on it and must be
 *    ordered by the caller.  The array starts zero-filled (static storage)
 *    and every call leaves its per-tile counters at zero again; after a call
 *    whose kernels timed out (LBQ_ETIMEOUT from lbq_device_status), call
 *    lbq_linear_fwd_noalloc_reset before the next call.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
lbq_status lbq_linear_fwd_noalloc(const void* X, int m, const lbq_qweight* q,
                                  const void* A, const void* B, int rank,
                                  float s, float* Y, float* T_save,
                                  lbq_stream_t stream);

/*
 * Zero the per-tile counters of lbq_linear_fwd_noalloc's array (an
 * asynchronous memset on `stream`; allocates nothing).  Needed only after a
 * call whose kernels timed out.  (No counterpart in the source pages.)
 */
lbq_status lbq_linear_fwd_noalloc_reset(lbq_stream_t stream);

/*
 * Several forwards with the same token count m in one call (for example the
 * seven linear layers of a transformer block at decode time, or q, k and v
 * sharing X).  Each problem is one lbq_linear_fwd: Y_i = X_i W_i^T +
 * s_i (X_i A_i^T) B_i^T with its own activations, weight, adapter and
 * outputs (same layouts, rank and alignment rules; `q` is a host pointer to
 * the descriptor).  For m <= 16 the problems run as one launch of the decode
 * GEMV per group of up to 8 weights (after one adapter launch per problem with
 * rank > 0), so the fixed costs of a launch are paid once per group.  For
 * larger m, when the problems' 128-row x token tiles together fill the
 * GPU's CTA slots, they run as grouped tensor-core launches of up to 8
 * problems each, without K splits; otherwise one after the other on
 * `stream`, each with its own K split.  The workspace
 * (lbq_linear_fwd_grouped_workspace_size bytes, zero-filled before its first
 * use, same reuse rules as lbq_linear_fwd's) serves all of them.  Results are
 * bit for bit those of separate lbq_linear_fwd calls on the same inputs when
 * the plan splits the matrices' work the same way; in every case each Y_i is
 * within the forward's stated bound and deterministic.  (The pages' forward,
 * QLoRA explainer, QLoRA技术原理, applied to a set of layers.)
 */
typedef struct {
    const void* X;            /* bf16 [m, q->k], device */
    const lbq_qweight* q;     /* host pointer to the weight descriptor */
    const void* A;            /* bf16 [rank, q->k], device, or NULL when rank == 0 */
    const void* B;            /* bf16 [q->n, rank], device, or NULL when rank == 0 */
    int32_t rank;             /* 0 .. 64 */
    float s;                  /* adapter scale */
    float* Y;                 /* fp32 [m, q->n], device */
    float* T_save;            /* fp32 [m, rank], device, or NULL when rank == 0 */
} lbq_fwd_problem;

size_t lbq_linear_fwd_grouped_workspace_size(int m, const lbq_fwd_problem* probs,
                                             int count);
lbq_status lbq_linear_fwd_grouped(int m, const lbq_fwd_problem* probs, int count,
                                  void* workspace, size_t workspace_bytes,
                                  lbq_stream_t stream);

/* The same forward for a channel-mix weight; Y columns in original order. */
size_t lbq_linear_fwd_mix_workspace_size(int m, const lbq_qweight_mix* q,
                                         int rank);
lbq_status lbq_linear_fwd_mix(const void* X, int m, const lbq_qweight_mix* q,
                              const void* A, const void* B, int rank, float s,
                              float* Y, float* T_save, void* workspace,
                              size_t workspace_bytes, lbq_stream_t stream);

/*
 * Several channel-mix forwards with the same token count m in one call (the
 * layers of a channel-mix model at decode time; GreenBit.AI article, 模型量化
 * (1): a bit width per output channel).  Each problem is one
 * lbq_linear_fwd_mix with its own activations, channel-mix weight (`q` is a
 * host pointer to the descriptor), adapter and outputs, under the same layout,
 * rank and alignment rules.  For m <= 16 both halves of every problem run as
 * decode GEMV launches of up to 8 weights each (after one adapter launch per
 * problem with rank > 0); for larger m the problems run one after the other
 * on `stream`.  The workspace (lbq_linear_fwd_mix_grouped_workspace_size
 * bytes, zero-filled before its first use, same reuse rules as
 * lbq_linear_fwd's) serves all of them.  Each Y_i is within the forward's
 * stated bound, in the original channel order, and deterministic.
 * Errors: LBQ_EINVAL (count < 1, m < 1, a NULL pointer, halves that are not
 * MinMax or differ in k), LBQ_EALIGN, LBQ_EWORKSPACE, as lbq_linear_fwd_mix.
 */
typedef struct {
    const void* X;              /* bf16 [m, k], device */
    const lbq_qweight_mix* q;   /* host pointer to the channel-mix descriptor */
    const void* A;              /* bf16 [rank, k], device, or NULL when rank == 0 */
    const void* B;              /* bf16 [n, rank] by original channel, or NULL */
    int32_t rank;               /* 0 .. 64 */
    float s;                    /* adapter scale */
    float* Y;                   /* fp32 [m, n] in the original channel order, device */
    float* T_save;              /* fp32 [m, rank], device, or NULL when rank == 0 */
} lbq_mix_problem;

size_t lbq_linear_fwd_mix_grouped_workspace_size(int m, const lbq_mix_problem* probs,
                                                 int count);
lbq_status lbq_linear_fwd_mix_grouped(int m, const lbq_mix_problem* probs, int count,
                                      void* workspace, size_t workspace_bytes,
                                      lbq_stream_t stream);

/*
 * Input gradient (QLoRA explainer, QLoRA技术原理: gradients pass through the
 * frozen quantized weight):
 *   U  = dY B  [m, rank]                         (fp32, written to U_save)
 *   dX = dY W + s U A  [m, k]                    (fp32)
 * dY bf16 [m, n].  Same rank, workspace and layout rules as lbq_linear_fwd.
 * Every weight format of lbq_qweight (MinMax INT4/INT2, the 4-bit codebook
 * with or without double quantization) is accepted; n must be a multiple of
 * 8.  The weight is dequantized to bf16 in the kernel: MinMax (code - zero)
 * in bf16 times the scale, codebook bf16(fp32(codebook[code] * absmax')).
 */
size_t lbq_linear_bwd_workspace_size(int m, const lbq_qweight* q, int rank);
lbq_status lbq_linear_bwd(const void* dY, int m, const lbq_qweight* q,
                          const void* A, const void* B, int rank, float s,
                          float* dX, float* U_save, void* workspace,
                          size_t workspace_bytes, lbq_stream_t stream);

/*
 * Several backward passes with the same token count m in one call (for
 * example the gate and up projections of an MLP block).  Each problem is one
 * lbq_linear_bwd: dX_i = dY_i W_i + s_i (dY_i B_i) A_i, with U_i = dY_i B_i
 * saved when rank_i > 0, with its own gradient, weight, adapter and outputs
 * (same layouts, rank and alignment rules; `q` is a host pointer to the
 * descriptor).  After one adapter launch per problem with rank > 0, when the
 * problems' 128-feature x token tiles together fill the GPU's CTA slots they
 * run as grouped tensor-core launches of up to 8 problems each, without
 * channel splits and needing no workspace; otherwise one after the other on
 * `stream`, each with the split its size calls for, sharing the workspace
 * (lbq_linear_bwd_grouped_workspace_size bytes, the largest of the
 * problems' lbq_linear_bwd_workspace_size; zero-filled before its first use,
 * same reuse rules).  Each dX_i is within the backward's stated bound and
 * deterministic.  Errors: those of lbq_linear_bwd for any problem, checked
 * before anything is launched; LBQ_EINVAL for m < 1, count < 1 or a NULL
 * probs.  (The pages' backward, QLoRA explainer, QLoRA技术原理, applied to a
 * set of layers.)
 */
typedef struct {
    const void* dY;           /* bf16 [m, q->n], device */
    const lbq_qweight* q;     /* host pointer to the weight descriptor */
    const void* A;            /* bf16 [rank, q->k], device, or NULL when rank == 0 */
    const void* B;            /* bf16 [q->n, rank], device, or NULL when rank == 0 */
    int32_t rank;             /* 0 .. 64 */
    float s;                  /* adapter scale */
    float* dX;                /* fp32 [m, q->k], device */
    float* U_save;            /* fp32 [m, rank], device, or NULL when rank == 0 */
} lbq_bwd_problem;

size_t lbq_linear_bwd_grouped_workspace_size(int m, const lbq_bwd_problem* probs,
                                             int count);
lbq_status lbq_linear_bwd_grouped(int m, const lbq_bwd_problem* probs, int count,
                                  void* workspace, size_t workspace_bytes,
                                  lbq_stream_t stream);

/*
 * Adapter gradients (the only trainable parameters; QLoRA explainer,
 * QLoRA技术原理):
 *   dA = s U^T X  [rank, k]       dB = s dY^T T  [n, rank]      (fp32)
 * X bf16 [m, k], dY bf16 [m, n], T = X A^T and U = dY B fp32 [m, rank] as
 * saved by lbq_linear_fwd / lbq_linear_bwd.  1 <= rank <= 64.
 */
lbq_status lbq_lora_grads(const void* X, const void* dY, int m, int n, int k,
                          const float* T, const float* U, int rank, float s,
                          float* dA, float* dB, lbq_stream_t stream);

/*
 * Channel-mix selection by sensitivity (GreenBit article, 模型量化 (1): the
 * bit width of each output channel follows how much quantizing it to fewer
 * bits costs).  W bf16 [n, k] (k % 128 == 0), calibration activations X bf16
 * [t, k], all device, 16-byte aligned.
 *   m2[j]    = (1/t) sum_i X[i,j]^2                       (fp64, i in order)
 *   e4, e2   = W_hat - W of the MinMax INT4 g128 / INT2 g64 quantization
 *              (lbq_quantize's arithmetic)
 *   score[c] = sum_j m2[j] (e2[c,j]^2 - e4[c,j]^2)          (fp64)
 * the rise of channel c's expected squared output error from INT4 to INT2.
 * The n4 channels with the highest score (the lower index first among equal
 * scores) are the INT4 channels: perm [n] (int32, device) lists them in
 * ascending order, then the others in ascending order -- the permutation of
 * lbq_qweight_mix.  score (fp64 [n], device) may be NULL.  workspace:
 * lbq_channel_mix_select_workspace_size(n, k) bytes of device memory (any
 * contents).  The per-channel sums run in an order of their own, so a score
 * may differ from a sequential fp64 sum in its last bits.
 */
size_t lbq_channel_mix_select_workspace_size(int n, int k);
lbq_status lbq_channel_mix_select(const void* W_bf16, int n, int k,
                                  const void* X_bf16, int t, int n4,
                                  double* score, int32_t* perm, void* workspace,
                                  size_t workspace_bytes, lbq_stream_t stream);

/*
 * out[i, :] = W[rows[i], :] for i < count: bf16 rows of W [n, k] (k % 8 ==
 * 0), for example the INT4 and INT2 halves of a channel-mix weight in the
 * order of its permutation.  rows: int32 device indices in [0, n).  (A data
 * movement helper; the pages have no counterpart.)
 */
lbq_status lbq_gather_rows(const void* W_bf16, int n, int k, const int32_t* rows,
                           int count, void* out, lbq_stream_t stream);

/*
 * Test hook for the bounded waits (no counterpart in the source pages): one
 * kernel waits on an mbarrier phase that never completes and then on a
 * device word that nothing sets, each for limit_us microseconds
 * (1 <= limit_us <= 1000000), then returns.  Each wait that gives up records
 * LBQ_ETIMEOUT in the device status word, exactly as the library's kernels do
 * when a wait runs out; lbq_device_status reads it.  Nothing traps or faults.
 */
lbq_status lbq_selftest_wait_timeout(uint32_t limit_us, lbq_stream_t stream);

/*
 * Device status word: the OR of the flags below recorded by kernels since the
 * last call (0 when none).  Synchronizes the current device, then clears the
 * word.  Returns LBQ_ECUDA if the read itself fails.
 */
#define LBQ_STATUS_TIMEOUT 1u      /* a bounded device-side wait gave up (LBQ_ETIMEOUT) */
#define LBQ_STATUS_BAD_TABLE 2u    /* a codebook broke the table preconditions */
lbq_status lbq_device_status(uint32_t* flags);

#ifdef __cplusplus
}
#endif
#endif /* LBQ_H */
