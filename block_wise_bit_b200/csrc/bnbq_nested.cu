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
// chunk whose index-order sum is exact (see absmax_chunk_sums) is added up in parallel.
#include "bnbq_device.cuh"
#include "bnbq_internal.h"

namespace bnbq {
namespace {

// min / max of an int over the CTA (every thread calls; every thread gets the result)
__device__ __forceinline__ int min_over_block(int v)
{
    __shared__ int r[32];
    for (int off = 16; off > 0; off >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, off));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) r[threadIdx.x >> 5] = v;
    __syncthreads();
    v = r[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); w++) v = min(v, r[w]);
    return v;
}

__device__ __forceinline__ int max_over_block(int v)
{
    return -min_over_block(-v);
}

// One CTA per chunk: the chunk is staged in shared memory with coalesced loads and summed in
// double.  The definition is the index-order sum, s = ((a0 + a1) + a2) + ...; when every partial
// sum of that order is exact the result does not depend on the order, and the CTA adds in
// parallel.  That holds when the ulps of the chunk's non-zero values span at most 2^17: every
// value is then an integer multiple of the smallest ulp U and below 2^24 times the largest, so
// the sum of at most 4096 = 2^12 of them stays below 2^(24+12+17) U = 2^53 U, an integer number
// of U's that a double holds exactly.  Otherwise (a wider spread, or a NaN or infinity) one thread
// adds in index order.
constexpr int kSumThreads = 256;

__device__ __forceinline__ int ulp_exponent(float x)  // biased exponent of x's ulp; 1 for subnormals
{
    const int e = (int)((__float_as_uint(x) >> 23) & 0xffu);
    return e == 0 ? 1 : e;
}

__global__ void __launch_bounds__(kSumThreads)
absmax_chunk_sums(const float* __restrict__ a, int64_t nb, double* __restrict__ work)
{
    __shared__ float chunk[kNestChunk];
    __shared__ double part[kSumThreads / 32];
    const int64_t start = (int64_t)blockIdx.x * kNestChunk;
    const int len = (int)((nb - start < kNestChunk) ? nb - start : kNestChunk);
    for (int i = threadIdx.x; i < len; i += blockDim.x) chunk[i] = __ldg(a + start + i);
    __syncthreads();
    // ulp exponent range of the non-zero values (a NaN or infinity forces the ordered sum)
    // (threads take every kSumThreads-th value: consecutive threads read consecutive words, so the
    // shared-memory reads never conflict; the exact sum below does not depend on the order)
    int emin = 255, emax = 0;
    for (int i = threadIdx.x; i < len; i += kSumThreads) {
        const float x = chunk[i];
        if (x == 0.0f) continue;
        const int e = ulp_exponent(x);
        emin = min(emin, e);
        emax = max(emax, (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u ? 1000 : e);
    }
    emin = __syncthreads_and(emin == 255) ? 0 : min_over_block(emin);
    emax = max_over_block(emax);
    const bool exact = emax - emin <= 17;
    if (exact) {  // every order gives the same (exact) sum
        double s = 0.0;
        for (int i = threadIdx.x; i < len; i += kSumThreads) s = __dadd_rn(s, (double)chunk[i]);
        for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
        if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int w = 0; w < kSumThreads / 32; w++) t = __dadd_rn(t, part[w]);
            work[blockIdx.x] = t;
        }
        return;
    }
    if (threadIdx.x != 0) return;
    double s = 0.0;
    for (int i = 0; i < len; i++) s = __dadd_rn(s, (double)chunk[i]);
    work[blockIdx.x] = s;
}

// The chunk sums in index order: the CTA stages them in shared memory with coalesced loads, a
// tile at a time, and one thread adds them up (the order is part of the definition).
constexpr int kFinishTile = 2048;

__global__ void __launch_bounds__(256)
absmax_mean_finish(const double* __restrict__ work, int64_t nchunks, int64_t nb, float* __restrict__ center)
{
    __shared__ double tile[kFinishTile];
    double total = 0.0;
    for (int64_t c0 = 0; c0 < nchunks; c0 += kFinishTile) {
        const int len = (int)(nchunks - c0 < kFinishTile ? nchunks - c0 : kFinishTile);
        __syncthreads();
        for (int i = threadIdx.x; i < len; i += blockDim.x) tile[i] = work[c0 + i];
        __syncthreads();
        if (threadIdx.x == 0)
            for (int i = 0; i < len; i++) total = __dadd_rn(total, tile[i]);
    }
    if (threadIdx.x == 0) *center = __double2float_rn(__ddiv_rn(total, (double)nb));
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
    const int64_t nchunks = (nb + kNestChunk - 1) / kNestChunk;
    absmax_chunk_sums<<<(unsigned)nchunks, 256, 0, s>>>(a, nb, work);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "absmax_chunk_sums launch");
    absmax_mean_finish<<<1, 256, 0, s>>>(work, nchunks, nb, center);
    return cuda_status(cudaGetLastError(), "absmax_mean_finish launch");
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
    return (int64_t)sizeof(double) * ((nb + kNestChunk - 1) / kNestChunk);
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
