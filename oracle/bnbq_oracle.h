/*
 * bnbq_oracle.h -- TEST INFRASTRUCTURE, NOT PART OF THE LIBRARY.
 *
 * A plain, slow, single-threaded CPU restatement of block-wise dynamic quantization of
 * optimizer state and of the 8-bit optimizer step built on it.  It exists only so that the
 * CUDA library can be checked against something written straight from the method's
 * description.  Only the test suite, the smoke check and the benchmark's CPU-baseline /
 * reference legs may load it.  It shares no code, header, table or constant with the CUDA
 * library (block_wise_bit_b200/csrc, include/bnbq.h) and never calls it.
 *
 * Sources, cited by key throughout this directory:
 *  [BWQ]   T. Dettmers, M. Lewis, S. Shleifer, L. Zettlemoyer, "8-bit Optimizers via
 *          Block-wise Quantization" (arXiv 2110.02861), abstract -- as reproduced on the page
 *          "Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略" (blog.csdn.net),
 *          section 2 "《通过块级量化的8位优化器》翻译与解读".
 *  [CN-32] same page, section "如果需要高精度的参数" (tensors with fewer than 4096 elements
 *          keep 32-bit state; min_8bit_size) and "更改单个参数的位数和其他超参数".
 *  [CN-OPT] page "bitsandbytes深度解析：PyTorch模型量化优化的完整实用指南" (agent.csdn.net),
 *          section "优化器模块深度分析" (AdamW8bit, Adam8bit, SGD8bit, Lion8bit, RMSprop8bit).
 *  [PT-W3] page "bitsandbytes - Quantização de LLM", section "Workflow 3: Otimizador 8-bit
 *          para treinamento eficiente em memória" (2 bytes of state per parameter).
 *  [NF4]   page "Bitsandbytes" (transformers docs, Turkish), section "Normal Float 4 (NF4)";
 *          page "Quantize 🤗 Transformers models", section "Using NF4 (Normal Float 4) data type".
 *  [ADAM]  D. Kingma, J. Ba, "Adam: A Method for Stochastic Optimization", Algorithm 1;
 *          I. Loshchilov, F. Hutter, "Decoupled Weight Decay Regularization", Algorithm 2.
 *  [LION]  X. Chen et al., "Symbolic Discovery of Optimization Algorithms", Algorithm 2 (Lion).
 *  [RMSP]  T. Tieleman, G. Hinton, "Lecture 6.5 -- rmsprop: divide the gradient by a running
 *          average of its recent magnitude", COURSERA: Neural Networks for Machine Learning,
 *          2012; eps added outside the square root and weight decay added to the gradient, as
 *          in torch.optim.RMSprop (no momentum, not centered).
 *  [QLORA] T. Dettmers et al., "QLoRA: Efficient Finetuning of Quantized LLMs", section 3
 *          (NormalFloat: quantiles of N(0,1), asymmetric 8+7 split with one shared zero;
 *          Double Quantization: the constants quantized again, 8-bit, blocks of 256, centred).
 *  [FP4]   page "Quantize 🤗 Transformers models", section "FP4 quantization" (4-bit loading with
 *          the FP4 data type); the format is the E2M1 4-bit float of the OCP Microscaling
 *          Formats (MX) specification v1.0, section 5.3.3.
 *  [NEST]  page "Bitsandbytes" (transformers docs, Turkish), section "İç içe nicelleştirme"
 *          (nested quantization: a second quantization of the already quantized weights'
 *          constants, about 0.4 bit per parameter saved).
 *
 * Floating point: IEEE binary32, round to nearest even, every operation rounded on its own
 * (built with -ffp-contract=off, no -ffast-math), division and sqrtf correctly rounded,
 * subnormals kept.  Scalars derived from the hyper-parameters are formed in double and
 * rounded once to float.  Per [BWQ]'s abstract only the stored optimizer statistics are 8-bit
 * and the optimizer is meant to behave as its 32-bit counterpart, so the update and every
 * quantization decision are taken in binary32.
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py against exact
 * rational arithmetic, scipy's normal distribution, or torch.optim; none is unpinned.
 */
#ifndef BNBQ_ORACLE_H
#define BNBQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* optimizer ids and dtype ids used by the oracle (its own numbering) */
enum { OR_ADAMW = 0, OR_ADAM = 1, OR_LION = 2, OR_MOMENTUM = 3, OR_RMSPROP = 4 };
enum { OR_F32 = 0, OR_BF16 = 1 };

typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
} oracle_hparams;

/* ---- codebooks (double precision construction, rounded once to binary32) ---- */
void oracle_code_dynamic_unsigned(float out[256]);
void oracle_code_dynamic_signed(float out[256]);
void oracle_code_nf4(float out[16]);
void oracle_code_fp4(float out[16]);
void oracle_code_linear(float out[256]);

/* mid_j of the nearest-code rule, j = 0..K-2 */
float oracle_code_mid(const float* code, int j);
/* q = #{ j : xn > mid_j }  (ties go to the lower code) */
int oracle_nearest_code(const float* code, int K, float xn);

/* bf16 helpers: exact widening, and round-to-nearest-even narrowing */
float oracle_bf16_to_f32(uint16_t h);
uint16_t oracle_f32_to_bf16(float f);

/*
 * Block-wise quantization of one tensor.  x holds n values of dtype x_dtype (OR_F32: float,
 * OR_BF16: uint16 bf16 bits).  Block b covers elements [b*B, min(n,(b+1)*B)).
 * absmax gets ceil(n/B) floats.  out gets n bytes (K == 256) or ceil(n/2) bytes (K == 16,
 * two 4-bit codes per byte, the even element in the high nibble).  Returns 0, or -1 on bad
 * arguments.
 */
int oracle_quantize_blockwise(const float* code, int K, const void* x, int x_dtype, int64_t n,
                              int B, float* absmax, uint8_t* out);

/* y_i = code[q_i] * absmax_b, written as float (OR_F32) or bf16 bits (OR_BF16). */
int oracle_dequantize_blockwise(const float* code, int K, const uint8_t* q, const float* absmax,
                                int64_t n, int B, void* y, int y_dtype);

/*
 * Nested (double) quantization of a block-scale array absmax[nb] [NEST]: offset = mean of the
 * scales (double sum over chunks of ORACLE_NEST_CHUNK, rounded once), then the centred scales
 * absmax_i - offset are quantized block-wise (blocks of ORACLE_NEST_B) with the 256-entry code2:
 * qabs[nb], absmax2[ceil(nb/ORACLE_NEST_B)].  Unnest rebuilds code2[qabs_i]*absmax2[i/256]+offset.
 */
#define ORACLE_NEST_B 256
#define ORACLE_NEST_CHUNK 4096
float oracle_absmax_mean(const float* absmax, int64_t nb);
int oracle_nest_absmax(const float* absmax, int64_t nb, const float* code2, uint8_t* qabs,
                       float* absmax2, float* offset);
int oracle_unnest_absmax(const uint8_t* qabs, const float* absmax2, float offset, const float* code2,
                         int64_t nb, float* out);

/*
 * One optimizer step on one tensor (t >= 1 is the step number, shared by all tensors).
 * state_bits == 8: s1 (and s2 for Adam/AdamW) are uint8 code indices, absmax1/absmax2 hold
 * ceil(n/B) block scales, code1 is the signed 256-entry code (m), code2 the unsigned one (v).
 * state_bits == 32: s1/s2 are float arrays, absmax and codes unused.
 * p is updated in place; g (dtype g_dtype) is read only.
 */
int oracle_step_tensor(int optim, int state_bits, float* p, const void* g, int g_dtype, int64_t n,
                       void* s1, void* s2, float* absmax1, float* absmax2, const float* code1,
                       const float* code2, int B, const oracle_hparams* hp, int t);

/* Same step restricted to blocks [b0, b1) of the tensor (used to time the oracle on a
 * bounded sample and to check sampled blocks of very large tensors). */
int oracle_step_blocks(int optim, int state_bits, float* p, const void* g, int g_dtype, int64_t n,
                       void* s1, void* s2, float* absmax1, float* absmax2, const float* code1,
                       const float* code2, int B, const oracle_hparams* hp, int t, int64_t b0,
                       int64_t b1);

#ifdef __cplusplus
}
#endif
#endif
