// bnbq_internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/bnbq.h"

namespace bnbq {

// Set the thread-local error text and return `st` (printf-style).
bnbq_status fail(bnbq_status st, const char* fmt, ...);
// Map a CUDA error to BNBQ_ECUDA with its text (cudaSuccess -> BNBQ_OK).
bnbq_status cuda_status(cudaError_t e, const char* what);
// BNBQ_EUNSUPPORTED if `s` is being captured into a CUDA graph (the step entry points refuse it).
bnbq_status refuse_capture(cudaStream_t s);

// BNBQ_OK if `bytes` bytes from `p` are device (or managed) memory of the current device, inside
// one allocation; else BNBQ_EINVAL naming `name`.  Used for codebooks before any launch.
bnbq_status check_device_array(const void* p, size_t bytes, const char* name);

// Device-side flag word of the current device (a __device__ variable; its address is taken
// once per device).
bnbq_status device_flag_ptr(unsigned** out);

// Number of SMs of the current device (cached per device).
bnbq_status sm_count(int* out);

// Kernel launchers (argument checks already done by the caller).
bnbq_status launch_quantize(const float* code, int K, const void* A, bnbq_dtype dt, int64_t n,
                            int B, float* absmax, uint8_t* out, cudaStream_t s);
bnbq_status launch_dequantize(const float* code, int K, const uint8_t* q, const float* absmax,
                              int64_t n, int B, void* out, bnbq_dtype dt, cudaStream_t s);

// Nested quantization of block scales: blocks of kNestBlock scales, the mean summed in double
// over chunks of kNestChunk scales.
constexpr int kNestBlock = 256;
constexpr int kNestChunk = 4096;
// absmax2/qabs <- block-wise quantization of a[i] - *center (fp32, blocks of kNestBlock).
bnbq_status launch_quantize_centred(const float* code2, const float* a, int64_t nb, const float* center,
                                    float* absmax2, uint8_t* qabs, cudaStream_t s);
// Dequantize with block scales code2[qabs_b] * absmax2[b / kNestBlock] + *center.
bnbq_status launch_dequantize_nested(const float* code, int K, const uint8_t* q, const uint8_t* qabs,
                                     const float* absmax2, const float* center, const float* code2, int64_t n,
                                     int B, void* out, bnbq_dtype dt, cudaStream_t s);
// *center <- mean of a[0..nb) (double chunk sums into work[ceil(nb/kNestChunk)], rounded once).
bnbq_status launch_absmax_mean(const float* a, int64_t nb, double* work, float* center, cudaStream_t s);
// out[i] <- code2[qabs_i] * absmax2[i / kNestBlock] + *center.
bnbq_status launch_unnest(const uint8_t* qabs, const float* absmax2, const float* center, const float* code2,
                          int64_t nb, float* out, cudaStream_t s);

// One entry of the device descriptor table used by the step kernel (64 bytes).
struct alignas(16) StepDesc {
    float* p;
    const void* g;
    void* s1;
    void* s2;
    float* a1;
    float* a2;
    int64_t n;
    int32_t first_block;  // global index of this tensor's first block
    int32_t flags;        // bit 0: g is bf16; bit 1: 8-bit state
};
static_assert(sizeof(StepDesc) == 64, "descriptor layout");
// The step kernel reads a descriptor as four 16-byte words (load_cur in bnbq_step.cu).
static_assert(offsetof(StepDesc, p) == 0 && offsetof(StepDesc, g) == 8 && offsetof(StepDesc, s1) == 16 &&
                  offsetof(StepDesc, s2) == 24 && offsetof(StepDesc, a1) == 32 && offsetof(StepDesc, a2) == 40 &&
                  offsetof(StepDesc, n) == 48 && offsetof(StepDesc, first_block) == 56 &&
                  offsetof(StepDesc, flags) == 60,
              "descriptor field offsets");
constexpr int32_t kDescGBf16 = 1;
constexpr int32_t kDescState8 = 2;

// Scalars of one step, derived on the host (double, rounded once to binary32).
struct StepScalars {
    float b1, b2, omb1, omb2;
    float step_size;     // lr / (1 - b1^t)
    float sqrt_bc2;      // sqrt(1 - b2^t)
    float rcp_sqrt_bc2;  // RN(1 / sqrt_bc2)
    float decay;         // 1 - lr*wd (AdamW, Lion) or 1
    float lr, eps, wd;
    int upd_fast;        // the FMA square root and division of the update may be used (see below)
};

// Host rule for StepScalars::upd_fast: the update's exact FMA square root and division need the
// denominator sqrt(v)/sqrt(1-b2^t) + eps (or sqrt(v) + eps) inside [2^-50, 2^63] whenever v lies in
// [2^-100, 2^100], which holds for 0 <= eps <= 2^60 and sqrt(1-b2^t) in [2^-12, 1].
inline bool update_fast_allowed(float eps, float sqrt_bc2)
{
    return eps >= 0.0f && eps <= 0x1p60f && sqrt_bc2 >= 0x1p-12f && sqrt_bc2 <= 1.0f;
}

bnbq_status launch_step(bnbq_optim opt, const StepDesc* d_table, int ntensors, int total_blocks,
                        const StepScalars& sc, const float* code1, const float* code2, int B,
                        cudaStream_t s);

}  // namespace bnbq
