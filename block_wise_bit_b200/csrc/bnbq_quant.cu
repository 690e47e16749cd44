// bnbq_quant.cu -- standalone block-wise quantize / dequantize kernels for sm_100a.
//
// Block-wise quantization ("8-bit Optimizers via Block-wise Quantization", abstract, quoted on
// the blog.csdn.net bitsandbytes guide, section 2): blocks of B consecutive elements are
// scaled by their own absolute maximum and quantized independently; here one group of threads
// owns one block (16 elements per thread for fp32 input, 32 for bf16, as 4-element chunks whose
// addresses are consecutive across the group, so every load and store is a coalesced vector
// access).
// NF4 packing (two 4-bit codes per byte) follows the 4-bit type of the page "Bitsandbytes",
// section "Normal Float 4 (NF4)".
//
// Roofline: HBM.  Quantize moves 4 (fp32) or 2 (bf16) bytes in and 1 (8-bit) or 0.5 (NF4)
// bytes out per element, plus 4 bytes per block; dequantize the reverse.  The grid is
// persistent: SMs x resident CTAs, each CTA striding over blocks.  Aligned fp32 input reaches
// the threads through shared memory: one bulk copy (cp.async.bulk, completed on an mbarrier)
// per 32 KB tile, two tiles ahead.
#include <float.h>
#include <stdlib.h>

#include <mutex>

#include "bnbq_async.cuh"
#include "bnbq_device.cuh"
#include "bnbq_internal.h"
#include "bnbq_search_fma.cuh"

namespace bnbq {
namespace {

constexpr int kQThreads = 512;

// Geometry of the quantize kernel.  A thread holds EPT elements of its group's block -- 16 for
// fp32 input, 32 for bf16, so that every thread has 64 bytes of input in flight -- as NCH chunks
// of CW consecutive elements (one vector load each: 4 fp32 or bf16, or 8 bf16 when WIDE); chunk
// j of thread tg starts at element CW * (j * G + tg) of the block, so a group's loads and stores
// are contiguous.
template <int B, bool BF16, bool WIDE>
struct QGeom {
    static constexpr int CW = WIDE ? 8 : 4;
    static constexpr int EPT = BF16 ? 32 : 16;
    static constexpr int NCH = EPT / CW;
    static constexpr int G = B / EPT;                  // threads per block-group
    static constexpr int kGroups = kQThreads / G;      // block-groups per CTA
    static constexpr int kGroupWarps = G >= 32 ? G / 32 : 1;
    static constexpr size_t kSmem = sizeof(CodeSmem) + sizeof(float) * kGroups * 2 * kGroupWarps;
    static_assert(G >= 1 && kQThreads % G == 0 && (!WIDE || BF16), "group geometry");
    // A CTA's blocks of one pass form a tile of kGroups * B elements (32 KB of input for either
    // dtype).  Staged variant (fp32 input): tiles are copied into shared memory one or two tiles
    // ahead of the threads; aligned bf16 input: the next tile is prefetched into L2.
    static constexpr int kES = BF16 ? 2 : 4;
    static constexpr int64_t kTileElems = (int64_t)kGroups * B;
    static constexpr uint32_t kTileBytes = (uint32_t)(kTileElems * kES);
    static constexpr size_t kStageOff = (kSmem + 127) / 128 * 128;
    static constexpr int kStages = 2;
    static constexpr size_t kBarOff = kStageOff + (size_t)kStages * kTileBytes;
    static constexpr size_t kSmemStaged = kBarOff + kStages * sizeof(uint64_t);
    // Chunk rotation of the staged reads: with fewer than 8 threads per block, thread tg of group
    // gi reads its chunks starting at chunk gi mod NCH, so that the 8 threads of each quarter-warp
    // phase of a 16-byte shared load fall in 8 different bank quads.
    static constexpr bool kRotate = G < 8;
    static_assert(kTileBytes % 16 == 0 && (!kRotate || (NCH & (NCH - 1)) == 0), "tile geometry");
};

template <bool BF16, int CW, bool FULL>
__device__ __forceinline__ void load_chunk(const void* A, int64_t e, int64_t n, float (&v)[CW])
{
    if (FULL || e + CW <= n) {
        if constexpr (BF16 && CW == 8) {
            const uint4 w = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(A) + e));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                v[2 * i] = bf16lo_to_f32(ws[i]);
                v[2 * i + 1] = bf16hi_to_f32(ws[i]);
            }
        } else if constexpr (BF16) {
            const uint2 w = ld_stream_u2(static_cast<const uint16_t*>(A) + e);
            v[0] = bf16lo_to_f32(w.x);
            v[1] = bf16hi_to_f32(w.x);
            v[2] = bf16lo_to_f32(w.y);
            v[3] = bf16hi_to_f32(w.y);
        } else {
            const float4 f = ld_stream_f4(static_cast<const float*>(A) + e);
            v[0] = f.x;
            v[1] = f.y;
            v[2] = f.z;
            v[3] = f.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < CW; i++) {
            float x = 0.0f;
            if (e + i < n) {
                if (BF16)
                    x = __uint_as_float((uint32_t)(static_cast<const uint16_t*>(A)[e + i]) << 16);
                else
                    x = static_cast<const float*>(A)[e + i];
            }
            v[i] = x;
        }
    }
}

// One 4-element fp32 chunk from a staged tile in shared memory (16-byte aligned).
__device__ __forceinline__ void load_chunk_smem(const unsigned char* p, float (&v)[4])
{
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
}

// Stage the codes (and, with_table, midpoints and bucket table) in shared memory.  Returns
// false, raising the flag once, if the codebook is invalid; `fast` = FMA quotient allowed;
// `general` = some bucket needs the general search.
__device__ bool stage_one_code(CodeSmem& cs, const float* code, int K, bool with_table, bool& fast,
                               bool& general, unsigned* flags)
{
    stage_code_pass1(cs, code, K);
    __syncthreads();
    bool bad = false, t = false;
    stage_code_pass2(cs, K, bad, t);
    bad = __syncthreads_or(bad);
    fast = !__syncthreads_or(t);
    if (bad) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(flags, kFlagBadCode);
        return false;
    }
    general = false;
    if (with_table) general = __syncthreads_or(stage_code_pass3(cs, K));
    return true;
}

// Nearest-code word of a normalised value in the kernel's search mode (code in the top byte).
template <int MODE>
__device__ __forceinline__ uint32_t code_word(const CodeSmem& cs, float x)
{
    if constexpr (MODE == kSearchPrefix11)
        return nearest_code_word11(cs.table, x);
    else if constexpr (MODE == kSearchSignedFma)  // measured 1.5-2% faster than kSearchSigned here
        return nearest_code_word_fma(cs.table + kHalf, x);
    else
        return nearest_code_word<MODE>(cs, x);
}

// The four nearest-code words of 4 consecutive elements.
template <int MODE, bool FAST>
__device__ __forceinline__ void words4(const CodeSmem& cs, const BlockScale& sc, const float* x, uint32_t (&w)[4])
{
    float2 x0 = make_float2(x[0], x[1]), x1 = make_float2(x[2], x[3]);
    if (FAST) {
        const float2 r = make_float2(sc.r, sc.r), na = make_float2(sc.na, sc.na);
        x0 = div2_rcp(x0, r, na);
        x1 = div2_rcp(x1, r, na);
    } else {
        x0 = make_float2(__fdiv_rn(x0.x, sc.a), __fdiv_rn(x0.y, sc.a));
        x1 = make_float2(__fdiv_rn(x1.x, sc.a), __fdiv_rn(x1.y, sc.a));
    }
    w[0] = code_word<MODE>(cs, x0.x);
    w[1] = code_word<MODE>(cs, x0.y);
    w[2] = code_word<MODE>(cs, x1.x);
    w[3] = code_word<MODE>(cs, x1.y);
}

// The codes of 4 consecutive elements, byte i = code of element i.
template <int MODE, bool FAST>
__device__ __forceinline__ uint32_t codes4(const CodeSmem& cs, const BlockScale& sc, const float* x)
{
    uint32_t w[4];
    words4<MODE, FAST>(cs, sc, x, w);
    return pack_top_bytes(w[0], w[1], w[2], w[3]);
}

// Four codes below 16, one per byte (c0 | c1 << 8 | c2 << 16 | c3 << 24), merged into nibble
// pairs: times 4097 adds a copy shifted left by 12 bits (no two nibbles overlap, so nothing
// carries), which puts c0 << 4 | c1 in byte 1 and c2 << 4 | c3 in byte 3.
__device__ __forceinline__ uint32_t nibble_pairs(uint32_t bytes4) { return bytes4 * 4097u; }

// The 4-bit codes of 4 consecutive elements packed two per byte (even element in the high nibble)
// in the low 16 bits.
template <int MODE, bool FAST>
__device__ __forceinline__ uint32_t nibbles4(const CodeSmem& cs, const BlockScale& sc, const float* x)
{
    return __byte_perm(nibble_pairs(codes4<MODE, FAST>(cs, sc, x)), 0u, 0x0031u);
}

// The same for 8 consecutive elements: four packed bytes.
template <int MODE, bool FAST>
__device__ __forceinline__ uint32_t nibbles8(const CodeSmem& cs, const BlockScale& sc, const float* x)
{
    return __byte_perm(nibble_pairs(codes4<MODE, FAST>(cs, sc, x)), nibble_pairs(codes4<MODE, FAST>(cs, sc, x + 4)),
                       0x7531u);
}

// Normalise, search and store one block's chunks (FAST: FMA quotient, else IEEE division; FULL:
// the block lies entirely inside the tensor, so no element needs a bounds check).
template <int B, bool BF16, bool WIDE, int K, int MODE, bool FAST, bool FULL>
__device__ __forceinline__ void quantize_store(const CodeSmem& cs, const BlockScale& sc,
                                               const float (&v)[QGeom<B, BF16, WIDE>::NCH][QGeom<B, BF16, WIDE>::CW],
                                               int64_t base, int tg, int64_t n, uint8_t* __restrict__ out, int rot)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr int G = Geo::G, CW = Geo::CW;
#pragma unroll
    for (int j = 0; j < Geo::NCH; j++) {
        const int64_t e = base + CW * (((j + rot) & (Geo::NCH - 1)) * G + tg);
        if (!FULL && e >= n) continue;
        if constexpr (K == 16) {
            if (FULL || e + CW <= n) {
                if constexpr (CW == 8)
                    st_stream_u32(out + (e >> 1), nibbles8<MODE, FAST>(cs, sc, &v[j][0]));
                else
                    *reinterpret_cast<uint16_t*>(out + (e >> 1)) = (uint16_t)nibbles4<MODE, FAST>(cs, sc, &v[j][0]);
                continue;
            }
        }
        uint32_t word[CW / 4];
#pragma unroll
        for (int h = 0; h < CW / 4; h++) word[h] = codes4<MODE, FAST>(cs, sc, &v[j][4 * h]);
        if (FULL || e + CW <= n) {
            if constexpr (K == 256 && CW == 8)
                st_stream_u2(out + e, make_uint2(word[0], word[1]));
            else
                st_stream_u32(out + e, word[0]);
        } else {  // the tensor's last, partial chunk: element by element
#pragma unroll
            for (int i = 0; i < CW; i++) {
                if (e + i >= n) break;
                const uint32_t c = (word[i >> 2] >> (8 * (i & 3))) & 0xffu;
                if constexpr (K == 256) {
                    out[e + i] = (uint8_t)c;
                } else if ((i & 1) == 0) {  // the high nibble; a missing partner leaves the low one 0
                    const uint32_t c1 = e + i + 1 < n ? (word[(i + 1) >> 2] >> (8 * ((i + 1) & 3))) & 0xffu : 0u;
                    out[(e + i) >> 1] = (uint8_t)((c << 4) | c1);
                }
            }
        }
    }
}

// One block held in registers (v[j] = chunk (j + rot) mod NCH of this thread): block absmax over
// the group, normalise, search, store.
// CENTER: quantize A[i] - off (one binary32 subtraction; fp32 input), the centred block scales of
// nested quantization.
template <int B, bool BF16, bool WIDE, int K, int MODE, bool CENTER, bool FULL>
__device__ __forceinline__ void quantize_values(const CodeSmem& cs, bool fast,
                                                float (&v)[QGeom<B, BF16, WIDE>::NCH][QGeom<B, BF16, WIDE>::CW],
                                                int64_t n, float* __restrict__ absmax, uint8_t* __restrict__ out,
                                                float* red, unsigned* flags, float off, int64_t b, int gi, int tg,
                                                int lane, unsigned gmask, int& parity, int rot)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr int G = Geo::G, CW = Geo::CW, NCH = Geo::NCH;
    const int64_t base = b * B;
    if constexpr (CENTER) {
#pragma unroll
        for (int j = 0; j < NCH; j++)
#pragma unroll
            for (int i = 0; i < CW; i++)
                if (FULL || base + CW * (((j + rot) & (NCH - 1)) * G + tg) + i < n) v[j][i] = __fsub_rn(v[j][i], off);
    }

    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; j++)
#pragma unroll
        for (int i = 0; i < CW; i += 2) m = max3_abs_nan(m, v[j][i], v[j][i + 1]);

    if constexpr (G <= 32) {
        m = group_max_nan<G>(m, gmask);
    } else {
        constexpr int W = G / 32;
        m = group_max_nan<32>(m, 0xffffffffu);
        float* r = red + (gi * 2 + parity) * W;
        if (lane == 0) r[tg >> 5] = m;
        group_barrier(1 + gi, G);
#pragma unroll
        for (int w = 0; w < W; w++) m = max_nan(m, r[w]);
        parity ^= 1;
    }
    if (tg == 0) {
        absmax[b] = m;
        if (!(m <= FLT_MAX)) atomicOr(flags, kFlagNonFinite);
    }
    const BlockScale sc = make_scale(m, fast);
    if (sc.fast)
        quantize_store<B, BF16, WIDE, K, MODE, true, FULL>(cs, sc, v, base, tg, n, out, rot);
    else
        quantize_store<B, BF16, WIDE, K, MODE, false, FULL>(cs, sc, v, base, tg, n, out, rot);
}

// One block read from global memory.
template <int B, bool BF16, bool WIDE, int K, int MODE, bool CENTER, bool FULL>
__device__ __forceinline__ void quantize_block(const CodeSmem& cs, bool fast, const void* __restrict__ A, int64_t n,
                                               float* __restrict__ absmax, uint8_t* __restrict__ out, float* red,
                                               unsigned* flags, float off, int64_t b, int gi, int tg, int lane,
                                               unsigned gmask, int& parity)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr int G = Geo::G, CW = Geo::CW, NCH = Geo::NCH;
    float v[NCH][CW];
#pragma unroll
    for (int j = 0; j < NCH; j++) load_chunk<BF16, CW, FULL>(A, b * B + CW * (j * G + tg), n, v[j]);
    quantize_values<B, BF16, WIDE, K, MODE, CENTER, FULL>(cs, fast, v, n, absmax, out, red, flags, off, b, gi, tg,
                                                          lane, gmask, parity, 0);
}

template <int B, bool BF16, bool WIDE, int K, int MODE, bool CENTER>
__device__ __forceinline__ void quantize_loop(const CodeSmem& cs, bool fast, const void* __restrict__ A, int64_t n,
                                              float* __restrict__ absmax, uint8_t* __restrict__ out, float* red,
                                              unsigned* flags, const float* __restrict__ center)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr int G = Geo::G;
    const int gi = threadIdx.x / G;
    const int tg = threadIdx.x % G;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G >= 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
    const int64_t nb = (n + B - 1) / B;
    const float off = CENTER ? __ldg(center) : 0.0f;
    int parity = 0;

    int64_t tile = blockIdx.x;  // the CTA's blocks of this pass: tile kGroups * tile .. + kGroups - 1
    for (int64_t b = (int64_t)blockIdx.x * Geo::kGroups + gi; b < nb; b += (int64_t)gridDim.x * Geo::kGroups) {
        if constexpr (BF16 && WIDE) {  // 16-byte aligned bf16: the CTA's next tile into L2 (a hint)
            const int64_t next = tile + gridDim.x;
            if (threadIdx.x == 0 && (next + 1) * Geo::kTileElems <= n)
                l2_prefetch(static_cast<const char*>(A) + next * (int64_t)Geo::kTileBytes, Geo::kTileBytes);
            tile = next;
        }
        if ((b + 1) * B <= n)  // group-uniform: every thread of the group holds the same block
            quantize_block<B, BF16, WIDE, K, MODE, CENTER, true>(cs, fast, A, n, absmax, out, red, flags, off, b, gi,
                                                                 tg, lane, gmask, parity);
        else
            quantize_block<B, BF16, WIDE, K, MODE, CENTER, false>(cs, fast, A, n, absmax, out, red, flags, off, b, gi,
                                                                  tg, lane, gmask, parity);
    }
}

// Staged loop (fp32 input, 16-byte aligned): the CTA's k-th tile is tile blockIdx.x + k *
// gridDim.x of the tensor (the blocks the plain loop would give it), copied into one of two
// shared-memory stages by a bulk copy that thread 0 issues two tiles ahead; the threads read
// their chunks from the stage, release it at a CTA barrier (after which thread 0 refills it) and
// quantize from registers.  Only whole tiles are staged; the partial last tile, if any, is
// quantized by the CTA whose turn it would be, with plain loads.  A copy that has not landed
// within the wait budget sets BNBQ_FLAG_TIMEOUT and ends the CTA (after a bounded wait for its
// copies still in flight).
template <int B, bool BF16, bool WIDE, int K, int MODE, bool CENTER>
__device__ __forceinline__ void quantize_loop_staged(const CodeSmem& cs, bool fast, const void* __restrict__ A,
                                                     int64_t n, float* __restrict__ absmax, uint8_t* __restrict__ out,
                                                     float* red, unsigned* flags, const float* __restrict__ center,
                                                     unsigned char* stage, uint64_t* full)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr int G = Geo::G, CW = Geo::CW, NCH = Geo::NCH;
    constexpr uint32_t TB = Geo::kTileBytes;
    static_assert(!BF16 && CW == 4, "staged input is fp32, 16-byte chunks");
    const int gi = threadIdx.x / G;
    const int tg = threadIdx.x % G;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G >= 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
    const int64_t nb = (n + B - 1) / B;
    const float off = CENTER ? __ldg(center) : 0.0f;
    const int rot = Geo::kRotate ? (gi & (NCH - 1)) : 0;
    int parity = 0;
    const int64_t ntiles = n / Geo::kTileElems;  // tiles that lie entirely inside the tensor
    const int64_t mine = ntiles > (int64_t)blockIdx.x ? (ntiles - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
    const unsigned char* src = static_cast<const unsigned char*>(A);
    auto tile_of = [&](int64_t k) { return (int64_t)blockIdx.x + k * (int64_t)gridDim.x; };
    if (threadIdx.x == 0) {
#pragma unroll
        for (int k = 0; k < Geo::kStages; k++) {
            if (k >= mine) break;
            mbar_arrive_expect(&full[k], TB);
            bulk_copy_g2s(stage + (size_t)k * TB, src + tile_of(k) * TB, TB, &full[k]);
        }
    }
    for (int64_t k = 0; k < mine; k++) {
        const int s = (int)(k & 1);
        const bool landed = mbar_wait(&full[s], (uint32_t)(k >> 1) & 1u);
        float v[NCH][CW];
        if (landed) {
            const unsigned char* t = stage + (size_t)s * TB + (size_t)gi * B * Geo::kES;
#pragma unroll
            for (int j = 0; j < NCH; j++)
                load_chunk_smem(t + (size_t)CW * (((j + rot) & (NCH - 1)) * G + tg) * Geo::kES, v[j]);
        }
        if (__syncthreads_or(!landed)) {  // CTA-uniform: stop, after the copies still in flight
            if (threadIdx.x == 0) {
                atomicOr(flags, kFlagTimeout);
                for (int64_t kk = k; kk < k + Geo::kStages && kk < mine; kk++)
                    (void)mbar_wait(&full[kk & 1], (uint32_t)(kk >> 1) & 1u);
            }
            return;
        }
        if (threadIdx.x == 0 && k + Geo::kStages < mine) {  // refill the released stage
            async_proxy_fence();
            mbar_arrive_expect(&full[s], TB);
            bulk_copy_g2s(stage + (size_t)s * TB, src + tile_of(k + Geo::kStages) * TB, TB, &full[s]);
        }
        quantize_values<B, BF16, WIDE, K, MODE, CENTER, true>(cs, fast, v, n, absmax, out, red, flags, off,
                                                              tile_of(k) * Geo::kGroups + gi, gi, tg, lane, gmask,
                                                              parity, rot);
    }
    if ((int64_t)blockIdx.x == ntiles % gridDim.x) {
        const int64_t b = ntiles * Geo::kGroups + gi;
        if (b < nb) {  // group-uniform
            if ((b + 1) * B <= n)
                quantize_block<B, BF16, WIDE, K, MODE, CENTER, true>(cs, fast, A, n, absmax, out, red, flags, off, b,
                                                                     gi, tg, lane, gmask, parity);
            else
                quantize_block<B, BF16, WIDE, K, MODE, CENTER, false>(cs, fast, A, n, absmax, out, red, flags, off, b,
                                                                      gi, tg, lane, gmask, parity);
        }
    }
}

template <int B, bool BF16, bool WIDE, int K, int MODE, bool CENTER, bool STAGED>
__device__ __forceinline__ void quantize_run(const CodeSmem& cs, bool fast, const void* __restrict__ A, int64_t n,
                                             float* __restrict__ absmax, uint8_t* __restrict__ out, float* red,
                                             unsigned* flags, const float* __restrict__ center, unsigned char* smem)
{
    using Geo = QGeom<B, BF16, WIDE>;
    if constexpr (STAGED)
        quantize_loop_staged<B, BF16, WIDE, K, MODE, CENTER>(cs, fast, A, n, absmax, out, red, flags, center,
                                                             smem + Geo::kStageOff,
                                                             reinterpret_cast<uint64_t*>(smem + Geo::kBarOff));
    else
        quantize_loop<B, BF16, WIDE, K, MODE, CENTER>(cs, fast, A, n, absmax, out, red, flags, center);
}

// STAGED: the input tiles come into shared memory by bulk copies (fp32 input, 16-byte aligned).
template <int B, bool BF16, bool WIDE, int K, bool CENTER, bool STAGED>
__global__ void __launch_bounds__(kQThreads, 2)
quantize_kernel(const float* __restrict__ code, const void* __restrict__ A, int64_t n,
                float* __restrict__ absmax, uint8_t* __restrict__ out, unsigned* flags,
                const float* __restrict__ center)
{
    using Geo = QGeom<B, BF16, WIDE>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    CodeSmem& cs = *reinterpret_cast<CodeSmem*>(smem_raw);
    float* red = reinterpret_cast<float*>(smem_raw + sizeof(CodeSmem));
    if constexpr (STAGED) {
        if (threadIdx.x == 0) {
            uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + Geo::kBarOff);
#pragma unroll
            for (int k = 0; k < Geo::kStages; k++) mbar_init(&full[k], 1);
            mbar_init_fence();
        }
        // (the codebook stage below synchronizes the CTA before any copy is issued)
    }
    bool fast, general;
    if constexpr (K == 16) {
        // 16 codes: the 11-bit-prefix table when no bucket of it holds two midpoints
        if (!stage_one_code(cs, code, K, false, fast, general, flags)) return;
        if (!__syncthreads_or(build_table11(cs.table, cs.mid, K))) {
            __syncthreads();
            quantize_run<B, BF16, WIDE, K, kSearchPrefix11, CENTER, STAGED>(cs, fast, A, n, absmax, out, red, flags,
                                                                            center, smem_raw);
            return;
        }
        __syncthreads();
        general = __syncthreads_or(stage_code_pass3(cs, K));
    } else if (!stage_one_code(cs, code, K, true, fast, general, flags)) {
        return;
    }
    if (general)
        quantize_run<B, BF16, WIDE, K, kSearchGeneral, CENTER, STAGED>(cs, fast, A, n, absmax, out, red, flags, center,
                                                                       smem_raw);
    else if (cs.code[0] >= 0.0f)  // every code >= 0
        quantize_run<B, BF16, WIDE, K, kSearchNonNeg, CENTER, STAGED>(cs, fast, A, n, absmax, out, red, flags, center,
                                                                      smem_raw);
    else {
        bias_negative_half(cs.table);  // the table is complete: the barrier of the general test above
        __syncthreads();
        quantize_run<B, BF16, WIDE, K, kSearchSignedFma, CENTER, STAGED>(cs, fast, A, n, absmax, out, red, flags,
                                                                         center, smem_raw);
    }
}

// code[nibble i of w] of a 16-entry codebook (nibble 0 = bits 0..3), its table offset formed by one
// shift and one mask.  The 16 codes sit in 16 different shared-memory banks, so these lookups
// never conflict (a table of code pairs indexed by the whole byte, read 8 bytes at a time,
// conflicted about three times per access).
__device__ __forceinline__ float code16_at(const float* code, uint32_t w, int i)
{
    const uint32_t off = (i == 0 ? (w << 2) : (w >> (4 * i - 2))) & 0x3cu;
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(code) + off);
}

// Dequantize: a lane's unit is 16 bytes of output (8 bf16 or 4 fp32 elements, always inside one
// block); consecutive lanes take consecutive units, so every load and store instruction of a warp
// covers one contiguous range.  One table lookup per element (for 4-bit codes the high nibble of
// a byte is the even element) and one packed product per pair.
// NESTED: the block scales are rebuilt from their nested quantization,
// A_b = code2[qabs_b] * absmax2[b / 256] + *center (two roundings), instead of read from absmax.
struct NestedScales {
    const uint8_t* qabs;
    const float* absmax2;
    const float* center;
    const float* code2;
};

constexpr int kDqUnits = 4;  // units per lane per span

template <bool BF16OUT>
struct DqGeom {
    static constexpr int kUnit = BF16OUT ? 8 : 4;      // elements per unit
    static constexpr int kSpan = 32 * kDqUnits * kUnit;
};

template <int K, int E>
struct DqWords {  // the unit's code bytes
    static constexpr int kBytes = K == 256 ? E : E / 2;
    static constexpr int kWords = (kBytes + 3) / 4;
};

template <int K, bool BF16OUT, bool NESTED>
__global__ void __launch_bounds__(256, (K == 16 && BF16OUT && !NESTED) ? 8 : (BF16OUT ? 6 : 5))
dequantize_kernel(const float* __restrict__ code, const uint8_t* __restrict__ q,
                  const float* __restrict__ absmax, int64_t n, int log2B, void* __restrict__ out,
                  unsigned* flags, NestedScales ns, bool out16, bool q4)
{
    using Geo = DqGeom<BF16OUT>;
    constexpr int UE = Geo::kUnit;
    using Wd = DqWords<K, UE>;
    __shared__ float code_s[NESTED ? 2 : 1][256];
    __shared__ float mid_s[NESTED ? 2 : 1][256];
    stage_codes(code_s[0], code, K);
    if constexpr (NESTED) stage_codes(code_s[NESTED ? 1 : 0], ns.code2, 256);
    __syncthreads();
    bool bad = false, tiny = false;
    stage_midpoints(code_s[0], mid_s[0], K, bad, tiny);
    if constexpr (NESTED) stage_midpoints(code_s[NESTED ? 1 : 0], mid_s[NESTED ? 1 : 0], 256, bad, tiny);
    if (__syncthreads_or(bad)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(flags, kFlagBadCode);
        return;
    }
    const float off = NESTED ? __ldg(ns.center) : 0.0f;
    // Unit j of a pass: fp32 output -- grid-stride units (a thread's units lie far apart);
    // bf16 output -- warp spans (a warp's units are one contiguous range).  Measured faster each
    // (warp spans for fp32 output: 3-11% slower).
    constexpr bool kSpans = BF16OUT;
    const int lane = threadIdx.x & 31;
    const int64_t nspans = (n + Geo::kSpan - 1) / Geo::kSpan;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t threads = (int64_t)gridDim.x * blockDim.x;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    auto unit_start = [&](int64_t span, int j) -> int64_t {
        if constexpr (kSpans) return span * Geo::kSpan + (int64_t)UE * (32 * j + lane);
        else return (int64_t)UE * (span * (kDqUnits * threads) + j * threads + gtid);
    };
    const int64_t first = kSpans ? (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5) : 0;
    const int64_t step = kSpans ? warps : 1;
    const int64_t npass = kSpans ? nspans : ((n + UE - 1) / UE + kDqUnits * threads - 1) / (kDqUnits * threads);
    for (int64_t span = first; span < npass; span += step) {
        uint32_t w[kDqUnits][Wd::kWords];
        float a[kDqUnits];
        // Nested scales in warp spans: the span's blocks are consecutive, so lane i rebuilds the
        // scale of the span's i-th block once and the lanes take theirs by shuffle (a span has at
        // most 32 blocks: blocks of at least 32 elements).  Measured 17% faster for NF4 weights at
        // blocksize 64; plain scales, one load per unit, were faster without the shuffle.
        constexpr bool kShare = NESTED && kSpans;
        float lane_scale = 0.0f;
        int64_t span_blk0 = 0;
        if constexpr (kShare) {
            span_blk0 = (span * Geo::kSpan) >> log2B;
            const int64_t blk = span_blk0 + lane;
            const int64_t nb = (n + (1ll << log2B) - 1) >> log2B;
            if (blk < nb && blk <= ((span + 1) * Geo::kSpan - 1) >> log2B)
                lane_scale = __fadd_rn(__fmul_rn(code_s[NESTED ? 1 : 0][__ldg(ns.qabs + blk)],
                                                 __ldg(ns.absmax2 + (blk >> 8))), off);
        }
#pragma unroll
        for (int j = 0; j < kDqUnits; j++) {
            const int64_t e = unit_start(span, j);
#pragma unroll
            for (int t = 0; t < Wd::kWords; t++) w[j][t] = 0;
            a[j] = 0.0f;
            if (e < n) {
                const uint8_t* qb = q + (K == 256 ? e : (e >> 1));
                if (e + UE <= n) {
                    if constexpr (Wd::kBytes == 2) {
                        w[j][0] = (uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(qb));
                    } else if constexpr (Wd::kBytes == 4 && K == 16) {  // codes 4- or 2-byte aligned
                        if (q4)
                            w[j][0] = ld_stream_u32(qb);
                        else
                            w[j][0] = (uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(qb)) |
                                      ((uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(qb + 2)) << 16);
                    } else {
#pragma unroll
                        for (int t = 0; t < Wd::kWords; t++) w[j][t] = ld_stream_u32(qb + 4 * t);
                    }
                } else {  // last, partial unit: bytes past the end read as code 0 and are not stored
                    const int nbytes = (int)(K == 256 ? n - e : (n - e + 1) / 2);
                    for (int i = 0; i < nbytes; i++) w[j][i >> 2] |= (uint32_t)qb[i] << (8 * (i & 3));
                }
                if constexpr (!kShare) {
                    const int64_t blk = e >> log2B;
                    if constexpr (NESTED)
                        a[j] = __fadd_rn(__fmul_rn(code_s[NESTED ? 1 : 0][__ldg(ns.qabs + blk)],
                                                   __ldg(ns.absmax2 + (blk >> 8))), off);
                    else
                        a[j] = __ldg(absmax + blk);
                }
            }
            if constexpr (kShare)  // every lane takes part (the source lane may hold no unit)
                a[j] = __shfl_sync(0xffffffffu, lane_scale, (int)((e >> log2B) - span_blk0) & 31);
        }
#pragma unroll
        for (int j = 0; j < kDqUnits; j++) {
            const int64_t e = unit_start(span, j);
            if (e >= n) continue;
            const float2 ap = make_float2(a[j], a[j]);
            float2 y[UE / 2];
#pragma unroll
            for (int h = 0; h < UE / 2; h++) {
                if constexpr (K == 256) {
                    const uint32_t wd = w[j][h >> 1];
                    const uint32_t b0 = 2u * (h & 1);
                    y[h] = mul2(make_float2(code_s[0][__byte_perm(wd, 0u, 0x4440u + b0)],
                                            code_s[0][__byte_perm(wd, 0u, 0x4441u + b0)]), ap);
                } else {  // byte h holds elements 2h (high nibble) and 2h+1 (low nibble)
                    y[h] = mul2(make_float2(code16_at(code_s[0], w[j][0], 2 * h + 1),
                                            code16_at(code_s[0], w[j][0], 2 * h)), ap);
                }
            }
            if (e + UE <= n) {
                if constexpr (BF16OUT) {
                    const uint4 v = make_uint4(pack_bf16x2(y[0].x, y[0].y), pack_bf16x2(y[1].x, y[1].y),
                                               pack_bf16x2(y[2].x, y[2].y), pack_bf16x2(y[3].x, y[3].y));
                    uint16_t* o = static_cast<uint16_t*>(out) + e;
                    if (out16) {
                        __stcs(reinterpret_cast<uint4*>(o), v);
                    } else {
                        st_stream_u2(o, make_uint2(v.x, v.y));
                        st_stream_u2(o + 4, make_uint2(v.z, v.w));
                    }
                } else {
                    st_stream_f4(static_cast<float*>(out) + e, make_float4(y[0].x, y[0].y, y[1].x, y[1].y));
                }
            } else {
                for (int i = 0; i < UE && e + i < n; i++) {
                    const float v = (i & 1) ? y[i >> 1].y : y[i >> 1].x;
                    if (BF16OUT)
                        static_cast<__nv_bfloat16*>(out)[e + i] = __float2bfloat16_rn(v);
                    else
                        static_cast<float*>(out)[e + i] = v;
                }
            }
        }
    }
}

template <typename Kern>
bnbq_status persistent_grid(Kern kern, int threads, size_t smem, int64_t work_units, int units_per_cta, int* grid)
{
    int sms = 0;
    bnbq_status st = sm_count(&sms);
    if (st != BNBQ_OK) return st;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (per_sm < 1) per_sm = 1;
    int64_t need = (work_units + units_per_cta - 1) / units_per_cta;
    int64_t g = (int64_t)sms * per_sm;
    *grid = (int)(need < g ? (need < 1 ? 1 : need) : g);
    return BNBQ_OK;
}

// Optional cap on the quantize grid (environment variable BNBQ_QUANT_MAX_CTAS, read at each
// launch; unset or not a positive integer = no cap): with few CTAs each one takes many tiles,
// which lets tests run the staged pipeline through many stage reuses at small sizes.
int quant_cta_cap()
{
    const char* v = getenv("BNBQ_QUANT_MAX_CTAS");
    if (!v || !*v) return 0;
    char* end = nullptr;
    const long c = strtol(v, &end, 10);
    return (end && *end == 0 && c > 0 && c < (1l << 30)) ? (int)c : 0;
}

// The size from which aligned fp32 input is staged: BNBQ_QUANT_STAGE_FROM=<elements> (read at
// each launch; a testing aid, e.g. 0 to stage every size) or the measured default.
int64_t quant_stage_from(int64_t dflt)
{
    const char* v = getenv("BNBQ_QUANT_STAGE_FROM");
    if (!v || !*v) return dflt;
    char* end = nullptr;
    const long long c = strtoll(v, &end, 10);
    return (end && *end == 0 && c >= 0) ? (int64_t)c : dflt;
}

template <int B, bool BF16, bool WIDE, int K, bool CENTER, bool STAGED>
bnbq_status launch_q_s(const float* code, const void* A, int64_t n, float* absmax, uint8_t* out,
                       cudaStream_t s, const float* center)
{
    using Geo = QGeom<B, BF16, WIDE>;
    constexpr size_t kSmem = STAGED ? Geo::kSmemStaged : Geo::kSmem;
    unsigned* flags = nullptr;
    bnbq_status st = device_flag_ptr(&flags);
    if (st != BNBQ_OK) return st;
    auto kern = quantize_kernel<B, BF16, WIDE, K, CENTER, STAGED>;
    // The kernel's shared-memory limit, set once per device (for this instantiation).
    constexpr int kDevs = 64;
    static std::mutex mu;
    static bool configured[kDevs] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kDevs) return fail(BNBQ_EUNSUPPORTED, "device ordinal %d", dev);
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!configured[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
            if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(quantize smem)");
            configured[dev] = true;
        }
    }
    int grid = 0;
    st = persistent_grid(kern, kQThreads, kSmem, (n + B - 1) / B, Geo::kGroups, &grid);
    if (st != BNBQ_OK) return st;
    const int cap = quant_cta_cap();
    if (cap > 0 && grid > cap) grid = cap;
    kern<<<grid, kQThreads, kSmem, s>>>(code, A, n, absmax, out, flags, center);
    return cuda_status(cudaGetLastError(), "quantize_kernel launch");
}

// Large aligned fp32 input: the staged kernel; otherwise plain loads.  Measured on B200 (blocksize
// 2048): with 8-bit codes staging is 1-3% faster from 2^26 elements on and up to 6% slower below
// (its first tiles wait for their copies); with 4-bit codes it is 2-3% faster at 2^28 but 5-7%
// slower at 2^27, hence the thresholds.  For bf16 input it lost 2-4% at every size: that kernel
// is bound by the shared-memory data pipe (the table lookups' bank conflicts) and the ALU rather
// than by load latency, and reading the stage back adds about 15% to the data pipe's wavefronts.
template <int B, bool BF16, bool WIDE, int K, bool CENTER = false>
bnbq_status launch_q(const float* code, const void* A, int64_t n, float* absmax, uint8_t* out,
                     cudaStream_t s, const float* center = nullptr)
{
    if constexpr (!BF16) {
        using Geo = QGeom<B, BF16, WIDE>;
        const int64_t from = quant_stage_from(K == 256 ? (1ll << 26) : (1ll << 28));
        if ((reinterpret_cast<uintptr_t>(A) & 15u) == 0 && n >= from && n >= Geo::kTileElems)
            return launch_q_s<B, BF16, WIDE, K, CENTER, true>(code, A, n, absmax, out, s, center);
    }
    return launch_q_s<B, BF16, WIDE, K, CENTER, false>(code, A, n, absmax, out, s, center);
}

// bf16 input 16-byte aligned, with codes aligned for 8 (8-bit) or 4 (4-bit) bytes per store:
// 8-element chunks, and thread 0 of each CTA prefetches the CTA's next 32 KB tile into L2 at the
// start of each pass (measured on B200 at 2^28 elements: 8-bit codes 4-7% faster, NF4 unchanged;
// two tiles ahead was slower for 8-bit codes); otherwise 4-element chunks.
template <int B, bool BF16>
bnbq_status launch_q_k(const float* code, int K, const void* A, int64_t n, float* absmax,
                       uint8_t* out, cudaStream_t s)
{
    const bool wide = BF16 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0 &&
                      (reinterpret_cast<uintptr_t>(out) & (K == 256 ? 7u : 3u)) == 0;
    if (wide)
        return K == 256 ? launch_q<B, true, true, 256>(code, A, n, absmax, out, s)
                        : launch_q<B, true, true, 16>(code, A, n, absmax, out, s);
    return K == 256 ? launch_q<B, BF16, false, 256>(code, A, n, absmax, out, s)
                    : launch_q<B, BF16, false, 16>(code, A, n, absmax, out, s);
}

template <int B>
bnbq_status launch_q_b(const float* code, int K, const void* A, bnbq_dtype dt, int64_t n,
                       float* absmax, uint8_t* out, cudaStream_t s)
{
    return dt == BNBQ_BF16 ? launch_q_k<B, true>(code, K, A, n, absmax, out, s)
                           : launch_q_k<B, false>(code, K, A, n, absmax, out, s);
}

template <int K, bool BF16OUT, bool NESTED = false>
bnbq_status launch_dq(const float* code, const uint8_t* q, const float* absmax, int64_t n, int B,
                      void* out, cudaStream_t s, NestedScales ns = NestedScales{})
{
    unsigned* flags = nullptr;
    bnbq_status st = device_flag_ptr(&flags);
    if (st != BNBQ_OK) return st;
    int log2B = 0;
    while ((1 << log2B) < B) log2B++;
    int grid = 0;
    auto kern = dequantize_kernel<K, BF16OUT, NESTED>;
    st = persistent_grid(kern, 256, 0, (n + DqGeom<BF16OUT>::kSpan - 1) / DqGeom<BF16OUT>::kSpan, 256 / 32, &grid);
    if (st != BNBQ_OK) return st;
    const bool out16 = (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
    const bool q4 = (reinterpret_cast<uintptr_t>(q) & 3u) == 0;
    kern<<<grid, 256, 0, s>>>(code, q, absmax, n, log2B, out, flags, ns, out16, q4);
    return cuda_status(cudaGetLastError(), "dequantize_kernel launch");
}

}  // namespace

bnbq_status launch_quantize(const float* code, int K, const void* A, bnbq_dtype dt, int64_t n,
                            int B, float* absmax, uint8_t* out, cudaStream_t s)
{
    switch (B) {
        case 64: return launch_q_b<64>(code, K, A, dt, n, absmax, out, s);
        case 128: return launch_q_b<128>(code, K, A, dt, n, absmax, out, s);
        case 256: return launch_q_b<256>(code, K, A, dt, n, absmax, out, s);
        case 2048: return launch_q_b<2048>(code, K, A, dt, n, absmax, out, s);
        case 4096: return launch_q_b<4096>(code, K, A, dt, n, absmax, out, s);
        default: return fail(BNBQ_EINVAL, "blocksize %d not in {64, 128, 256, 2048, 4096}", B);
    }
}

bnbq_status launch_quantize_centred(const float* code2, const float* a, int64_t nb, const float* center,
                                    float* absmax2, uint8_t* qabs, cudaStream_t s)
{
    return launch_q<kNestBlock, false, false, 256, true>(code2, a, nb, absmax2, qabs, s, center);
}

bnbq_status launch_dequantize_nested(const float* code, int K, const uint8_t* q, const uint8_t* qabs,
                                     const float* absmax2, const float* center, const float* code2, int64_t n,
                                     int B, void* out, bnbq_dtype dt, cudaStream_t s)
{
    const NestedScales ns{qabs, absmax2, center, code2};
    if (K == 256)
        return dt == BNBQ_BF16 ? launch_dq<256, true, true>(code, q, nullptr, n, B, out, s, ns)
                               : launch_dq<256, false, true>(code, q, nullptr, n, B, out, s, ns);
    return dt == BNBQ_BF16 ? launch_dq<16, true, true>(code, q, nullptr, n, B, out, s, ns)
                           : launch_dq<16, false, true>(code, q, nullptr, n, B, out, s, ns);
}

bnbq_status launch_dequantize(const float* code, int K, const uint8_t* q, const float* absmax,
                              int64_t n, int B, void* out, bnbq_dtype dt, cudaStream_t s)
{
    if (K == 256)
        return dt == BNBQ_BF16 ? launch_dq<256, true>(code, q, absmax, n, B, out, s)
                               : launch_dq<256, false>(code, q, absmax, n, B, out, s);
    return dt == BNBQ_BF16 ? launch_dq<16, true>(code, q, absmax, n, B, out, s)
                           : launch_dq<16, false>(code, q, absmax, n, B, out, s);
}

}  // namespace bnbq
