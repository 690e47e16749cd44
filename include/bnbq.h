/*
 * bnbq.h -- C ABI of the block-wise 8-bit optimizer-state library for NVIDIA B200 (sm_100a).
 *
 * The method: "8-bit Optimizers via Block-wise Quantization" (Dettmers, Lewis, Shleifer,
 * Zettlemoyer; arXiv 2110.02861), whose abstract is reproduced on the page
 * "Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略" (blog.csdn.net), section 2
 * "《通过块级量化的8位优化器》翻译与解读".  Stateful optimizers keep per-parameter statistics
 * (momentum's smoothed gradient sum, Adam's smoothed sum and squared sum); the abstract stores
 * them in 8 bits by block-wise quantization -- the tensor is cut into blocks that are quantized
 * independently, each in parallel -- with a dynamic (non-linear) code whose relative error
 * stays small across many orders of magnitude.  NF4 is the 16-value 4-bit type of the page "Bitsandbytes"
 * (transformers docs), section "Normal Float 4 (NF4)".
 *
 * Conventions for every entry point:
 *  - Pointers named as device memory must point to memory of the current CUDA device; host
 *    structs are read before the call returns and not kept.  The caller owns every buffer.
 *    Codebook pointers are checked before anything is launched: one that is not device (or
 *    managed) memory of the current device, or whose codes would run past the end of its
 *    allocation as the driver reports it, returns BNBQ_EINVAL.
 *  - Work is enqueued on `stream` (NULL = the legacy default stream) and is asynchronous with
 *    respect to the host.  Argument checks are synchronous: a non-OK status means nothing was
 *    enqueued.  BNBQ_ECUDA means a CUDA call failed; the CUDA error text is in bnbq_last_error().
 *  - No entry point aborts, throws, traps or waits on the device.  A codebook that fails the
 *    device-side check (strictly increasing, finite, within [-1, 1]) makes the kernel write
 *    nothing and sets BNBQ_FLAG_BAD_CODE; non-finite values met while building block scales set
 *    BNBQ_FLAG_NONFINITE.  Kernels wait only for their own bulk copies into shared memory, each
 *    wait bounded (about a second); one that runs out sets BNBQ_FLAG_TIMEOUT.  Read the flags
 *    with bnbq_device_flags().
 *  - Blocks have `blocksize` consecutive elements -- 64, 128, 256, 2048 or 4096 for quantize and
 *    dequantize, 256, 2048 or 4096 for the optimizer step; the last block of a tensor may be
 *    shorter; blocks never span two tensors.  Block b's scale is absmax[b].
 *  - Alignment (checked; BNBQ_EINVAL if violated): fp32 arrays and fp32 state 16 bytes, bf16
 *    arrays 8 bytes, 8-bit codes 4 bytes, packed 4-bit codes 2 bytes, absmax and codebooks 4
 *    bytes; the nested-scale entry points state their own.
 */
#ifndef BNBQ_H
#define BNBQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BNBQ_API __attribute__((visibility("default")))
#else
#define BNBQ_API
#endif

/* Same type as cudaStream_t, declared here so this header needs no CUDA include. */
typedef struct CUstream_st* bnbq_stream_t;

typedef enum {
    BNBQ_OK = 0,
    BNBQ_EINVAL = 1,       /* an argument is out of range, null, or misaligned */
    BNBQ_EUNSUPPORTED = 2, /* a valid request this library version does not handle */
    BNBQ_ECUDA = 3         /* a CUDA runtime call failed (see bnbq_last_error) */
} bnbq_status;

typedef enum { BNBQ_F32 = 0, BNBQ_BF16 = 1 } bnbq_dtype;

typedef enum {
    BNBQ_ADAMW = 0,   /* Adam with decoupled weight decay (two states: m signed, v unsigned) */
    BNBQ_ADAM = 1,    /* Adam, weight decay added to the gradient (two states) */
    BNBQ_LION = 2,     /* Lion: one signed state */
    BNBQ_MOMENTUM = 3, /* SGD with momentum, dampening 0: one signed state */
    BNBQ_RMSPROP = 4   /* RMSprop: one state, the running mean of squares (unsigned code) */
} bnbq_optim;

typedef enum {
    BNBQ_CODE_DYNAMIC_SIGNED = 0,   /* 256 values, for m / Lion / momentum state */
    BNBQ_CODE_DYNAMIC_UNSIGNED = 1, /* 256 values, for Adam's v and RMSprop's state */
    BNBQ_CODE_NF4 = 2,              /* 16 values */
    BNBQ_CODE_LINEAR = 3,           /* 256 values, -1 + 2k/255 */
    BNBQ_CODE_FP4 = 4               /* 16 values: E2M1 4-bit float / 6, the -0 pattern as +0.25/6 */
} bnbq_code_kind;

/* device flag bits (bnbq_device_flags) */
#define BNBQ_FLAG_BAD_CODE 0x1u  /* a codebook failed the device-side check; the kernel wrote nothing */
#define BNBQ_FLAG_NONFINITE 0x2u /* a block scale (absmax) came out NaN or Inf */
#define BNBQ_FLAG_TIMEOUT 0x4u   /* a kernel's bounded wait for its own copy ran out; its outputs are incomplete */

/*
 * Block-wise quantization (abstract of "8-bit Optimizers via Block-wise Quantization";
 * NF4: "Bitsandbytes", section "Normal Float 4 (NF4)").
 *   code      device, code_size fp32 values, strictly increasing, within [-1, 1]
 *   code_size 256 (8-bit codes, one byte per element) or 16 (two 4-bit codes per byte)
 *   A         device, n elements of a_dtype
 *   blocksize 64, 128, 256, 2048 or 4096 (64 is the 4-bit weight setting of QLoRA)
 *   absmax    device, out: ceil(n/blocksize) fp32, absmax[b] = max |A_i| over block b
 *   out       device, out: n bytes (code_size 256) or ceil(n/2) bytes (code_size 16; element 2k
 *             in the high nibble of byte k, element 2k+1 in the low nibble; for odd n the last
 *             low nibble is 0)
 * Element i of block b gets q = #{ j : A_i/absmax[b] > mid_j } with
 * mid_j = fl32((code_j + code_{j+1})/2): the nearest code, a tie going to the lower code; a
 * block whose absmax is 0 maps to the code nearest 0.  The division is correctly rounded.
 * n == 0 is a no-op.  Testing aids, read at each call: BNBQ_QUANT_MAX_CTAS=<k> caps the kernel's
 * grid at k CTAs (every CTA then takes many tiles; unset = one or two CTAs per SM);
 * BNBQ_QUANT_STAGE_FROM=<n> stages aligned fp32 input into shared memory from n elements on
 * (unset = from 2^26 for 256 codes, 2^28 for 16).
 */
BNBQ_API bnbq_status bnbq_quantize_blockwise(const float* code, int code_size, const void* A,
                                    bnbq_dtype a_dtype, int64_t n, int blocksize, float* absmax,
                                    uint8_t* out, bnbq_stream_t stream);

/*
 * Block-wise dequantization: out_i = code[q_i] * absmax[b] (one fp32 rounding; bf16 output is
 * that value rounded to nearest even).  q layout as bnbq_quantize_blockwise's `out`.
 *   out  device, n elements of out_dtype.  n == 0 is a no-op.
 */
BNBQ_API bnbq_status bnbq_dequantize_blockwise(const float* code, int code_size, const uint8_t* q,
                                      const float* absmax, int64_t n, int blocksize, void* out,
                                      bnbq_dtype out_dtype, bnbq_stream_t stream);

/*
 * Nested (double) quantization of a block-scale array (page "Bitsandbytes", section "İç içe
 * nicelleştirme": a second quantization of the quantized weights' constants, about 0.4 bit per
 * parameter saved; scheme of "QLoRA: Efficient Finetuning of Quantized LLMs", section 3, Double
 * Quantization).  For absmax[nb] (fp32, >= 0, e.g. from bnbq_quantize_blockwise):
 *   offset    device, out: 1 fp32, the mean of absmax -- a double sum over chunks of 4096
 *             consecutive scales (each chunk in index order, then the chunk sums in index
 *             order), divided by nb in double and rounded once; 0 when nb == 0
 *   qabs      device, out: nb bytes, absmax2 device, out: ceil(nb/256) fp32 -- the block-wise
 *             8-bit quantization (blocks of 256, code2) of absmax_i - offset (one fp32
 *             subtraction), with the rule of bnbq_quantize_blockwise
 *   code2     device, 256 fp32 (the signed dynamic code is the intended one)
 *   workspace device, bnbq_nested_workspace_bytes(nb) bytes, 8-byte aligned, caller-owned;
 *             its contents are scratch.  absmax must be 16-byte aligned.
 * Asynchronous on `stream`; a 4-byte memset of the workspace and two kernel launches.
 */
BNBQ_API int64_t bnbq_nested_workspace_bytes(int64_t nb);
BNBQ_API bnbq_status bnbq_quantize_absmax_nested(const float* absmax, int64_t nb, const float* code2,
                                                 uint8_t* qabs, float* absmax2, float* offset,
                                                 void* workspace, bnbq_stream_t stream);

/* Rebuild the scales: absmax_out[i] = code2[qabs_i] * absmax2[i/256] + *offset (two fp32
 * roundings, multiply then add).  All pointers device memory. */
BNBQ_API bnbq_status bnbq_dequantize_absmax_nested(const uint8_t* qabs, const float* absmax2,
                                                   const float* offset, const float* code2, int64_t nb,
                                                   float* absmax_out, bnbq_stream_t stream);

/* bnbq_dequantize_blockwise with each block's scale rebuilt on the fly from its nested
 * quantization (as bnbq_dequantize_absmax_nested computes it): one pass, no fp32 scale array. */
BNBQ_API bnbq_status bnbq_dequantize_blockwise_nested(const float* code, int code_size, const uint8_t* q,
                                                      const uint8_t* qabs, const float* absmax2,
                                                      const float* offset, const float* code2, int64_t n,
                                                      int blocksize, void* out, bnbq_dtype out_dtype,
                                                      bnbq_stream_t stream);

/* One tensor of a multi-tensor optimizer step.  All pointers are device memory. */
typedef struct {
    float* p;         /* n fp32 parameters, updated in place */
    const void* g;    /* n gradients of g_dtype, read only */
    void* state1;     /* m (Adam/AdamW), Lion or momentum state: uint8[n] codes or fp32[n] */
    void* state2;     /* v (Adam/AdamW only): uint8[n] or fp32[n]; ignored otherwise */
    float* absmax1;   /* ceil(n/blocksize) block scales of state1 (state_bits 8 only) */
    float* absmax2;   /* ceil(n/blocksize) block scales of state2 (Adam/AdamW, 8-bit only) */
    int64_t n;        /* elements; 0 = skip this entry */
    int32_t g_dtype;  /* bnbq_dtype of g */
    int32_t state_bits; /* 8: quantized state; 32: plain fp32 state (small tensors, embeddings) */
} bnbq_tensor;

/* Hyper-parameters as torch.optim names them.  Momentum SGD reads beta1 as its momentum;
 * Lion reads beta1 (update interpolation) and beta2 (state decay); RMSprop reads beta1 as its
 * smoothing constant alpha. */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
} bnbq_hparams;

/*
 * One fused optimizer step over a list of tensors, in one kernel launch ("dequantize -> 32-bit
 * update -> requantize" per block, as the abstract of "8-bit Optimizers via Block-wise
 * Quantization" describes 8-bit statistics with 32-bit optimizer performance; optimizer list
 * from "bitsandbytes深度解析", section "优化器模块深度分析"; tensors that keep 32-bit state:
 * "Py之bitsandbytes…详细攻略", section "如果需要高精度的参数").
 *   opt         bnbq_optim
 *   list        host array of ntensors descriptors (0 <= ntensors <= 1<<20)
 *   hp          host pointer; all values finite; for Adam/AdamW 0 <= beta1, beta2 < 1; for
 *               RMSprop 0 <= beta1 < 1
 *   step        t >= 1, the 1-based step number shared by all tensors (Adam bias correction)
 *   code1       device, 256 fp32: code for state1 (needed if any tensor is 8-bit): the signed
 *               code, or for RMSprop the unsigned one
 *   code2       device, 256 fp32: unsigned code for Adam/AdamW state2 (else may be NULL)
 *   blocksize   256, 2048 or 4096
 * Per element, in binary32 with every operation rounded on its own:
 *   AdamW: m = b1*m + (1-b1)*g; v = b2*v + ((1-b2)*g)*g; p = p*(1-lr*wd);
 *          p = p - (lr/(1-b1^t)) * (m / (sqrt(v)/sqrt(1-b2^t) + eps))
 *   Adam:  g = g + wd*p (if wd != 0), then AdamW's rule without the p*(1-lr*wd) factor
 *   Lion:  c = b1*m + (1-b1)*g; p = p*(1-lr*wd) - lr*sign(c); m = b2*m + (1-b2)*g
 *   Momentum: g = g + wd*p (if wd != 0); m = b1*m + g; p = p - lr*m
 *   RMSprop: g = g + wd*p (if wd != 0); v = b1*v + ((1-b1)*g)*g; p = p - lr * (g / (sqrt(v) + eps))
 *          (T. Tieleman, G. Hinton, "Lecture 6.5 -- rmsprop", 2012; eps outside the root, as in
 *          torch.optim.RMSprop without momentum; the pages name RMSprop8bit in
 *          "bitsandbytes深度解析", section "优化器模块深度分析")
 * (scalar factors such as 1-b1, lr/(1-b1^t) are formed in double on the host and rounded once.)
 * For 8-bit state the old state is code[q]*absmax[b]; after the update each block gets a new
 * absmax = max|state| and the state is requantized by the nearest-code rule above.
 * The library keeps a small per-device cache of uploaded descriptor tables keyed by the list's
 * contents (freed by bnbq_release); a list seen before needs no upload.
 * A stream that is being captured into a CUDA graph is refused with BNBQ_EUNSUPPORTED before
 * anything is enqueued: the bias corrections of `step` are kernel arguments and the descriptor
 * table is rewritten or evicted by later calls, so a replayed capture would not be this call.
 */
BNBQ_API bnbq_status bnbq_step_8bit(bnbq_optim opt, const bnbq_tensor* list, int ntensors,
                           const bnbq_hparams* hp, int step, const float* code1,
                           const float* code2, int blocksize, bnbq_stream_t stream);

/*
 * bnbq_step_8bit_noalloc: the same step as bnbq_step_8bit (same arguments, same results) for
 * callers that cannot let a library allocate device memory -- code whose device memory all
 * belongs to its own pool or arena, processes that must not grow their footprint after start-up,
 * or step loops that must never reach an allocator.  The pages describe no such entry point; it
 * is this library's own.  Instead of an allocated, cached descriptor table it uses a fixed table
 * compiled into the library: at most 4096 non-empty tensors per call (256 KiB of device memory
 * on every GPU that loads the library, kept until the process exits); a longer list returns
 * BNBQ_EINVAL.  It calls no cudaMalloc, cudaFree or other allocating routine.  The first call on
 * each device looks up the table's device address; with CUDA's lazy module loading that lookup may
 * load the library's device code, which is when the table (and the code) take device memory.  A
 * caller that must not allocate later should make one call on each device at start-up, before
 * capturing any stream.  Like bnbq_step_8bit it refuses a stream that is being captured
 * (BNBQ_EUNSUPPORTED).  All calls on a
 * device share the one table and each call rewrites the entries it uses: calls whose work can
 * overlap on the GPU (different streams with no ordering between them) race on it, so order them.
 */
BNBQ_API bnbq_status bnbq_step_8bit_noalloc(bnbq_optim opt, const bnbq_tensor* list, int ntensors,
                                            const bnbq_hparams* hp, int step, const float* code1,
                                            const float* code2, int blocksize, bnbq_stream_t stream);

/* Host-side codebook construction (out: host memory, 256 or 16 floats per bnbq_code_size).
 * Returns the number of values written, or -1 for an unknown kind / NULL out. */
BNBQ_API int bnbq_codebook(bnbq_code_kind kind, float* out);
BNBQ_API int bnbq_code_size(bnbq_code_kind kind);

/* Host-side check of a codebook in host memory: BNBQ_OK if K in {16, 256}, every value finite,
 * within [-1, 1] and strictly increasing; else BNBQ_EINVAL with the reason. */
BNBQ_API bnbq_status bnbq_check_codebook(const float* host_code, int K);

/* Read (and if `clear`, reset) the calling device's flag word.  Synchronizes the device. */
BNBQ_API bnbq_status bnbq_device_flags(uint32_t* out, int clear);

/* Thread-local text for the last non-OK status returned on this thread ("" if none). */
BNBQ_API const char* bnbq_last_error(void);

/* Free the cached descriptor tables of all devices (waits for kernels that use them). */
BNBQ_API void bnbq_release(void);

/* Library version, e.g. "0.1.0". */
BNBQ_API const char* bnbq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BNBQ_H */
