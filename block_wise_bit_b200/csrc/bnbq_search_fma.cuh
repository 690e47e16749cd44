// bnbq_search_fma.cuh -- the signed nearest-code search with the sign handled on the FMA pipe.
//
// Same rule and same results as nearest_code_word<kSearchSigned> (bnbq_device.cuh): a bucket per
// 16-bit prefix of |x|, the entry holding the midpoints below the bucket in its top byte and the
// bucket's threshold in its low half, so that a carry into the top byte decides the one midpoint
// inside the bucket.  Here the negative half's entries are raised by kNegBias = 0xffff once the
// table is built: entry - low16(x) then equals the unbiased entry plus the complement
// 0xffff - low16(x), so entry + low16(x) * (+1 or -1) gives the code for either sign with one
// integer multiply-add, and the sign half's offset is a multiply-add too -- work for the FMA pipe
// instead of logic operations on the integer pipe, which quantize keeps busier.
#pragma once

#include "bnbq_device.cuh"

namespace bnbq {

constexpr int kSearchSignedFma = 5;
constexpr uint32_t kNegBias = 0xffffu;

// Raise the negative half, entries [0, kHalf) of the table (index -kHalf .. -1 from its centre);
// all threads of the CTA, between barriers.
__device__ __forceinline__ void bias_negative_half(uint32_t* table)
{
    for (int i = threadIdx.x; i < kHalf; i += blockDim.x) table[i] += kNegBias;
}

// Nearest code of x (code in the top byte; low bytes scratch); `center` = the biased table's
// entry of index 0.
__device__ __forceinline__ uint32_t nearest_code_word_fma(const uint32_t* center, float x)
{
    const uint32_t xb = __float_as_uint(x);
    const int32_t sx = (int32_t)xb >> 31;                                    // -1 if x < 0, else 0
    const uint32_t t = __float_as_uint(fmaxf(fabsf(x), kTinyEdge));         // magnitude (NaN -> 2^-26)
    const int32_t off = (int32_t)((t >> 14) & 0x3ffcu) + sx * (4 * kHalf);  // 4 * [-kHalf, kHalf)
    const uint32_t e = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(center) + off);
    return e + (xb & 0xffffu) * (uint32_t)(2 * sx + 1);
}

}  // namespace bnbq
