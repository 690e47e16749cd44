// Exhaustive checks of the exact FMA square root and quotients of bnbq_device.cuh against CUDA's
// correctly rounded __fsqrt_rn / __fdiv_rn:
//   sqrt    sqrt2_ranged(v) for every binary32 v in [2^-100, 2^100] (both lanes of the pair);
//   quot    div2_rcp(a, RN(1/b), -b), the one-correction quotient used for the block
//           normalisation, the division by sqrt(1-b2^t) and the update's m/den, for every pair of
//           significands a, b in [1, 2) (2^46 pairs), with RN(1/b) from rcp_rn_scaled_range as
//           the kernels form it.  Scaling a and b by powers of two scales every intermediate
//           exactly while the remainder stays exact and the quotient normal, so this covers every
//           exponent pair in that range; the reciprocal itself is checked over its whole range by
//           reciprocal_exhaustive.cu;
//   ranged  div2_ranged(a, b) (reciprocal formed inside) on 2^32 pairs drawn by a counter-based
//           hash over the kernels' operand ranges: |a| in [2^-60, 2^60], b in [2^-50, 2^63].
// Prints one line per check and exits 0 only if every count is 0.
#include <cstdint>
#include <cstdio>

#include "../../block_wise_bit_b200/csrc/bnbq_device.cuh"

__global__ void sqrt_check(unsigned long long* bad)
{
    const uint32_t lo = 0x0D800000u, hi = 0x71800000u;  // bit patterns of 2^-100 and 2^100
    const uint32_t total = hi - lo + 1;
    unsigned long long n = 0;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (total + 1) / 2; i += gridDim.x * blockDim.x) {
        const uint32_t b0 = lo + 2 * i, b1 = b0 + 1 <= hi ? b0 + 1 : b0;
        const float2 v = make_float2(__uint_as_float(b0), __uint_as_float(b1));
        const float2 s = bnbq::sqrt2_ranged(v);
        n += __float_as_uint(s.x) != __float_as_uint(__fsqrt_rn(v.x));
        n += __float_as_uint(s.y) != __float_as_uint(__fsqrt_rn(v.y));
    }
    if (n) atomicAdd(bad, n);
}

// One thread per significand of b (bi0 + thread index); a runs over all 2^23 significands, two per pair.
__global__ void quot_check(uint32_t bi0, unsigned long long* bad)
{
    const uint32_t bi = bi0 + blockIdx.x * blockDim.x + threadIdx.x;
    const float b = __uint_as_float(0x3f800000u | bi);
    const float2 r = make_float2(bnbq::rcp_rn_scaled_range(b), bnbq::rcp_rn_scaled_range(b));
    const float2 nb = make_float2(-b, -b);
    unsigned long long n = 0;
    for (uint32_t ai = 0; ai < (1u << 23); ai += 2) {
        const float2 a = make_float2(__uint_as_float(0x3f800000u | ai), __uint_as_float(0x3f800000u | (ai + 1)));
        const float2 q = bnbq::div2_rcp(a, r, nb);
        n += __float_as_uint(q.x) != __float_as_uint(__fdiv_rn(a.x, b));
        n += __float_as_uint(q.y) != __float_as_uint(__fdiv_rn(a.y, b));
    }
    if (n) atomicAdd(bad, n);
}

__device__ __forceinline__ uint32_t mix(uint32_t x)
{  // 32-bit finaliser of MurmurHash3 (Appleby), a bijection used as a counter-based generator
    x ^= x >> 16; x *= 0x85ebca6bu; x ^= x >> 13; x *= 0xc2b2ae35u; x ^= x >> 16;
    return x;
}

__device__ __forceinline__ float draw(uint32_t h, int e_lo, int e_hi, bool sign)
{
    const uint32_t e = (uint32_t)(e_lo + 127) + (h >> 23) % (uint32_t)(e_hi - e_lo);
    return __uint_as_float((sign && (h & 0x100u) ? 0x80000000u : 0u) | (e << 23) | (mix(h) & 0x7fffffu));
}

__global__ void ranged_check(uint32_t k0, unsigned long long* bad)
{
    unsigned long long n = 0;
    const uint32_t k = k0 + blockIdx.x * blockDim.x + threadIdx.x;
    for (uint32_t j = 0; j < 64; j++) {
        const uint32_t c = (k << 6) | j;
        const float2 a = make_float2(draw(mix(2 * c), -60, 60, true), draw(mix(2 * c + 1), -60, 60, true));
        const float2 b = make_float2(draw(mix(c ^ 0x9e3779b9u), -50, 63, false), draw(mix(c ^ 0x7f4a7c15u), -50, 63, false));
        const float2 q = bnbq::div2_ranged(a, b);
        n += __float_as_uint(q.x) != __float_as_uint(__fdiv_rn(a.x, b.x));
        n += __float_as_uint(q.y) != __float_as_uint(__fdiv_rn(a.y, b.y));
    }
    if (n) atomicAdd(bad, n);
}

int main()
{
    unsigned long long* d = nullptr;
    if (cudaMalloc(&d, 3 * sizeof(*d)) != cudaSuccess) return 2;
    cudaMemset(d, 0, 3 * sizeof(*d));
    sqrt_check<<<148 * 16, 256>>>(d);
    cudaError_t e = cudaDeviceSynchronize();
    for (uint32_t c = 0; c < 64 && e == cudaSuccess; c++) {  // 2^17 significands of b per launch
        quot_check<<<(1u << 17) / 128, 128>>>(c << 17, d + 1);
        e = cudaDeviceSynchronize();
    }
    for (uint32_t c = 0; c < 16 && e == cudaSuccess; c++) {  // 2^22 threads x 64 pairs x 16 launches = 2^32
        ranged_check<<<(1u << 22) / 256, 256>>>(c << 22, d + 2);
        e = cudaDeviceSynchronize();
    }
    unsigned long long h[3] = {~0ull, ~0ull, ~0ull};
    cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost);
    printf("sqrt status %s mismatches %llu\n", cudaGetErrorString(e), h[0]);
    printf("quot status %s mismatches %llu\n", cudaGetErrorString(e), h[1]);
    printf("ranged status %s mismatches %llu\n", cudaGetErrorString(e), h[2]);
    return (e == cudaSuccess && h[0] == 0 && h[1] == 0 && h[2] == 0) ? 0 : 1;
}
