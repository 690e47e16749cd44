// bnbq_nested.cu -- nested (double) quantization of block scales.
//
// Page "Bitsandbytes" (transformers docs, Turkish), section "İç içe nicelleştirme": a second
// quantization of the already quantized weights' constants, saving about 0.4 bit per parameter.
// Following the double quantization of "QLoRA: Efficient Finetuning of Quantized LLMs" (section
// 3): the fp32 block scales (all >= 0) are centred by their mean and quantized block-wise to 8
// bits in blocks of kNestBlock = 256 with a signed 256-entry code; a scale is rebuilt as
// code2[qabs_b] * absmax2[b / 256] + offset.  With 4-bit weights in blocks of 64 this stores
// 8/64 + 32/(64*256) bits per weight for the scales instead of 32/64.
//
// The mean is a plain double sum in a fixed order -- chunks of kNestChunk consecutive scales,
// each summed in index order, then the chunk sums in index order -- divided by nb in double and
// rounded once to binary32, so every run (and the CPU restatement) gets the same offset.  A
// chunk whose index-order sum is exact is added up in parallel, and so are the chunk sums when the
// whole array's sum is exact (absmax_mean_kernel).
#include "bnbq_device.cuh"
#include "bnbq_internal.h"

namespace bnbq {
namespace {

// The mean in one launch.  One CTA per chunk of kNestChunk scales; each thread takes every
// kMeanThreads-th value of the chunk (coalesced loads, kept in registers) and forms, in one pass,
// the range of the values' ulp exponents and their double sum.  The definition is the index-order
// sum, s = ((a0 + a1) + a2) + ...; when every partial sum of that order is exact the result does
// not depend on the order, and the CTA adds in parallel.  That holds when the ulps of the chunk's
// non-zero values span at most 2^17: every value is then an integer multiple of the smallest ulp U
// and below 2^24 times the largest, so the sum of at most 4096 = 2^12 of them stays below
// 2^(24+12+17) U = 2^53 U, an integer number of U's that a double holds exactly.  Otherwise (a
// wider spread, or a NaN or infinity) one thread adds the chunk in index order.
// Each CTA stores its chunk sum and exponent range, and the last CTA to finish (a counter in the
// workspace, zeroed before the launch) adds the chunk sums: in parallel when the sum over the
// whole array is exact by the same argument -- nb values whose ulps span at most 2^d, with
// nb * 2^(24+d) <= 2^53 -- else in index order by one thread.  No CTA waits for another.
constexpr int kMeanThreads = 256;
constexpr int kMeanWarps = kMeanThreads / 32;
constexpr int kPerThread = kNestChunk / kMeanThreads;
constexpr int kNoValue = 255;      // exponent-range sentinel: no non-zero value
constexpr int kNotFinite = 1000;   // exponent of a NaN or infinity: forces the ordered sums

__device__ __forceinline__ int ulp_exponent(float x)  // biased exponent of x's ulp; 1 for subnormals
{
    const int e = (int)((__float_as_uint(x) >> 23) & 0xffu);
    return e == 0 ? 1 : (e == 0xff ? kNotFinite : e);
}

// CTA-wide min of lo, max of hi and sum of s; every thread gets the results.
__device__ __forceinline__ void cta_reduce(int& lo, int& hi, double& s)
{
    __shared__ int rlo[kMeanWarps], rhi[kMeanWarps];
    __shared__ double rs[kMeanWarps];
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
    __syncthreads();  // the arrays may still be read from a previous call
    if ((threadIdx.x & 31) == 0) {
        rlo[threadIdx.x >> 5] = lo;
        rhi[threadIdx.x >> 5] = hi;
        rs[threadIdx.x >> 5] = s;
    }
    __syncthreads();
    lo = rlo[0];
    hi = rhi[0];
    s = rs[0];
    for (int w = 1; w < kMeanWarps; w++) {
        lo = min(lo, rlo[w]);
        hi = max(hi, rhi[w]);
        s = __dadd_rn(s, rs[w]);
    }
}

__device__ __forceinline__ bool sum_is_exact(int lo, int hi, int log2_count)
{
    return lo == kNoValue || (hi < kNotFinite && hi - lo + 24 + log2_count <= 53);
}

__global__ void __launch_bounds__(kMeanThreads)
absmax_mean_kernel(const float* __restrict__ a, int64_t nb, double* __restrict__ sums, int2* __restrict__ range,
                   unsigned* __restrict__ counter, float* __restrict__ center)
{
    __shared__ bool last;
    const int64_t start = (int64_t)blockIdx.x * kNestChunk;
    const int len = (int)((nb - start < kNestChunk) ? nb - start : kNestChunk);
    int lo = kNoValue, hi = 0;
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < kPerThread; k++) {
        const int i = (int)threadIdx.x + k * kMeanThreads;
        if (i < len) {
            const float x = __ldg(a + start + i);
            if (x != 0.0f) {
                const int e = ulp_exponent(x);
                lo = min(lo, e);
                hi = max(hi, e);
            }
            s = __dadd_rn(s, (double)x);
        }
    }
    cta_reduce(lo, hi, s);
    if (threadIdx.x == 0) {
        if (!sum_is_exact(lo, hi, 12)) {  // the chunk in index order
            s = 0.0;
            for (int i = 0; i < len; i++) s = __dadd_rn(s, (double)__ldg(a + start + i));
        }
        sums[blockIdx.x] = s;
        range[blockIdx.x] = make_int2(lo, hi);
        __threadfence();
        last = atomicAdd(counter, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!last) return;
    // the last CTA: every other CTA's chunk sum and range are written (fence before the count)
    __threadfence();
    const int nchunks = (int)gridDim.x;
    lo = kNoValue;
    hi = 0;
    s = 0.0;
    for (int c = threadIdx.x; c < nchunks; c += kMeanThreads) {
        const int2 r = __ldcg(range + c);
        lo = min(lo, r.x);
        hi = max(hi, r.y);
        s = __dadd_rn(s, __ldcg(sums + c));
    }
    cta_reduce(lo, hi, s);
    if (threadIdx.x == 0) {
        int log2_nb = 0;
        while ((1ll << log2_nb) < nb) log2_nb++;
        if (!sum_is_exact(lo, hi, log2_nb)) {  // the chunk sums in index order
            s = 0.0;
            for (int c = 0; c < nchunks; c++) s = __dadd_rn(s, __ldcg(sums + c));
        }
        *center = __double2float_rn(__ddiv_rn(s, (double)nb));
    }
}

__global__ void __launch_bounds__(256)
unnest_kernel(const uint8_t* __restrict__ qabs, const float* __restrict__ absmax2, const float* __restrict__ center,
              const float* __restrict__ code2, int64_t nb, float* __restrict__ out)
{
    __shared__ float code_s[256];
    for (int j = threadIdx.x; j < 256; j += blockDim.x) code_s[j] = code2[j];
    __syncthreads();
    const float off = __ldg(center);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __fadd_rn(__fmul_rn(code_s[qabs[i]], __ldg(absmax2 + i / kNestBlock)), off);
}

int blocks_for(int64_t units, int threads)
{
    int sms = 148;
    sm_count(&sms);
    const int64_t need = (units + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(need < 1 ? 1 : (need < cap ? need : cap));
}

bool aligned_n(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

bnbq_status launch_absmax_mean(const float* a, int64_t nb, double* work, float* center, cudaStream_t s)
{
    // work: nchunks chunk sums (double), nchunks exponent ranges (int2), the finish counter
    const int64_t nchunks = (nb + kNestChunk - 1) / kNestChunk;
    int2* range = reinterpret_cast<int2*>(work + nchunks);
    unsigned* counter = reinterpret_cast<unsigned*>(range + nchunks);
    cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_status(e, "mean counter reset");
    absmax_mean_kernel<<<(unsigned)nchunks, kMeanThreads, 0, s>>>(a, nb, work, range, counter, center);
    return cuda_status(cudaGetLastError(), "absmax_mean_kernel launch");
}

bnbq_status launch_unnest(const uint8_t* qabs, const float* absmax2, const float* center, const float* code2,
                          int64_t nb, float* out, cudaStream_t s)
{
    unnest_kernel<<<blocks_for(nb, 256), 256, 0, s>>>(qabs, absmax2, center, code2, nb, out);
    return cuda_status(cudaGetLastError(), "unnest_kernel launch");
}

}  // namespace bnbq

using namespace bnbq;

extern "C" BNBQ_API int64_t bnbq_nested_workspace_bytes(int64_t nb)
{
    if (nb <= 0) return 0;
    const int64_t nchunks = (nb + kNestChunk - 1) / kNestChunk;
    return (int64_t)(sizeof(double) + sizeof(int2)) * nchunks + 8;  // sums, exponent ranges, counter
}

extern "C" BNBQ_API bnbq_status bnbq_quantize_absmax_nested(const float* absmax, int64_t nb, const float* code2,
                                                            uint8_t* qabs, float* absmax2, float* offset,
                                                            void* workspace, bnbq_stream_t stream)
{
    if (nb < 0) return fail(BNBQ_EINVAL, "nb = %lld < 0", (long long)nb);
    if (!code2 || !offset) return fail(BNBQ_EINVAL, "code2 and offset must be non-NULL");
    if (!aligned_n(code2, 4) || !aligned_n(offset, 4)) return fail(BNBQ_EINVAL, "code2 / offset not 4-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (nb == 0) return cuda_status(cudaMemsetAsync(offset, 0, sizeof(float), s), "offset = 0");
    if (!absmax || !qabs || !absmax2 || !workspace)
        return fail(BNBQ_EINVAL, "absmax, qabs, absmax2 and workspace must be non-NULL");
    if (!aligned_n(absmax, 16)) return fail(BNBQ_EINVAL, "absmax not 16-byte aligned");
    if (!aligned_n(qabs, 4)) return fail(BNBQ_EINVAL, "qabs not 4-byte aligned");
    if (!aligned_n(absmax2, 4)) return fail(BNBQ_EINVAL, "absmax2 not 4-byte aligned");
    if (!aligned_n(workspace, 8)) return fail(BNBQ_EINVAL, "workspace not 8-byte aligned");
    bnbq_status st = check_device_array(code2, 256 * sizeof(float), "code2");
    if (st != BNBQ_OK) return st;
    st = launch_absmax_mean(absmax, nb, static_cast<double*>(workspace), offset, s);
    if (st != BNBQ_OK) return st;
    return launch_quantize_centred(code2, absmax, nb, offset, absmax2, qabs, s);
}

extern "C" BNBQ_API bnbq_status bnbq_dequantize_absmax_nested(const uint8_t* qabs, const float* absmax2,
                                                              const float* offset, const float* code2, int64_t nb,
                                                              float* absmax_out, bnbq_stream_t stream)
{
    if (nb < 0) return fail(BNBQ_EINVAL, "nb = %lld < 0", (long long)nb);
    if (nb == 0) return BNBQ_OK;
    if (!qabs || !absmax2 || !offset || !code2 || !absmax_out)
        return fail(BNBQ_EINVAL, "qabs, absmax2, offset, code2 and absmax_out must be non-NULL");
    if (!aligned_n(absmax2, 4) || !aligned_n(offset, 4) || !aligned_n(code2, 4) || !aligned_n(absmax_out, 4))
        return fail(BNBQ_EINVAL, "absmax2, offset, code2 and absmax_out must be 4-byte aligned");
    bnbq_status st = check_device_array(code2, 256 * sizeof(float), "code2");
    if (st != BNBQ_OK) return st;
    return launch_unnest(qabs, absmax2, offset, code2, nb, absmax_out, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" BNBQ_API bnbq_status bnbq_dequantize_blockwise_nested(const float* code, int code_size, const uint8_t* q,
                                                                 const uint8_t* qabs, const float* absmax2,
                                                                 const float* offset, const float* code2, int64_t n,
                                                                 int blocksize, void* out, bnbq_dtype out_dtype,
                                                                 bnbq_stream_t stream)
{
    if (!code || !code2) return fail(BNBQ_EINVAL, "code and code2 must be non-NULL");
    if (code_size != 256 && code_size != 16) return fail(BNBQ_EINVAL, "code_size %d not in {16, 256}", code_size);
    if (!aligned_n(code, 4) || !aligned_n(code2, 4)) return fail(BNBQ_EINVAL, "codebooks not 4-byte aligned");
    if (n < 0) return fail(BNBQ_EINVAL, "n = %lld < 0", (long long)n);
    if (blocksize != 64 && blocksize != 128 && blocksize != 256 && blocksize != 2048 && blocksize != 4096)
        return fail(BNBQ_EINVAL, "blocksize %d not in {64, 128, 256, 2048, 4096}", blocksize);
    if (out_dtype != BNBQ_F32 && out_dtype != BNBQ_BF16) return fail(BNBQ_EINVAL, "out_dtype %d unknown", (int)out_dtype);
    if (n == 0) return BNBQ_OK;
    if (!q || !qabs || !absmax2 || !offset || !out) return fail(BNBQ_EINVAL, "q, qabs, absmax2, offset and out must be non-NULL");
    if (!aligned_n(q, code_size == 256 ? 4 : 2)) return fail(BNBQ_EINVAL, "q not %d-byte aligned", code_size == 256 ? 4 : 2);
    if (!aligned_n(absmax2, 4) || !aligned_n(offset, 4)) return fail(BNBQ_EINVAL, "absmax2 / offset not 4-byte aligned");
    const uintptr_t oa = out_dtype == BNBQ_BF16 ? 8 : 16;
    if (!aligned_n(out, oa)) return fail(BNBQ_EINVAL, "out not %d-byte aligned", (int)oa);
    bnbq_status st = check_device_array(code, sizeof(float) * (size_t)code_size, "code");
    if (st == BNBQ_OK) st = check_device_array(code2, 256 * sizeof(float), "code2");
    if (st != BNBQ_OK) return st;
    return launch_dequantize_nested(code, code_size, q, qabs, absmax2, offset, code2, n, blocksize, out, out_dtype,
                                    reinterpret_cast<cudaStream_t>(stream));
}
