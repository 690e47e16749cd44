// bnbq_step.cu -- the fused multi-tensor 8-bit optimizer step for sm_100a.
//
// Method ("8-bit Optimizers via Block-wise Quantization", abstract, quoted on the blog.csdn.net
// bitsandbytes guide, section 2): optimizer statistics are kept in 8 bits with block-wise
// dynamic quantization while the update runs at 32-bit precision.  Per block this kernel
//   loads p (fp32), g (fp32/bf16), the 8-bit codes and the block scales        (a4)
//   dequantizes m = code1[q1]*a1 and v = code2[q2]*a2 from shared memory         (a4)
//   applies the fp32 AdamW / Adam / Lion / momentum / RMSprop update, stores p    (a5)
//   reduces the new block absmax of each state across the block's thread group     (a6)
//   requantizes each state against its new absmax (nearest code) and stores it     (a7)
// Tensors that keep 32-bit state (fewer than 4096 elements, and embedding tables: page
// "Py之bitsandbytes…详细攻略", section "如果需要高精度的参数") are stepped by the same launch (a8).
//
// Layout and scheduling (a9): one launch per step for the whole tensor list.  The host uploads
// a table of tensor descriptors (cached across steps); blocks are numbered globally, tensor by
// tensor.  A persistent grid of kThreads-thread CTAs strides over them; a CTA holds
// kThreads/(B/kEPT) block-groups of B/kEPT threads, each group owning one block at a time with
// kEPT elements per thread (4-element chunks, consecutive across the group: every global access
// is a fully coalesced vector access).  Groups synchronise with their own named barrier, so the
// codebook tables are staged once per CTA and shared by all groups.  Each group walks the
// descriptor table with a monotone cursor and keeps the current tensor's fields in registers.
// Full blocks run without bounds checks; the last, partial block of a tensor takes a guarded path.
//
// Roofline: HBM.  AdamW with 8-bit state and bf16 gradients moves 14 bytes per element
// (p read+write 8, g 2, q1 and q2 read+write 4) plus 16 bytes per block of scales.
#include <float.h>
#include <limits.h>

#include <mutex>

#include "bnbq_device.cuh"
#include "bnbq_internal.h"

#ifndef BNBQ_STEP_EPT
#define BNBQ_STEP_EPT 16
#endif
#ifndef BNBQ_STEP_THREADS
#define BNBQ_STEP_THREADS 1024       // CTA size for blocksize 256 and 4096
#endif
#ifndef BNBQ_STEP_THREADS_2048
#define BNBQ_STEP_THREADS_2048 768   // CTA size for blocksize 2048 (80 registers: no spills)
#endif
#ifndef BNBQ_STEP_MIN_CTAS
#define BNBQ_STEP_MIN_CTAS 1
#endif

namespace bnbq {
namespace {

constexpr int kEPT = BNBQ_STEP_EPT;   // elements per thread per block
constexpr int kNCH = kEPT / 4;        // 4-element chunks per thread
static_assert(kEPT % 4 == 0, "whole chunks");

template <int B>
struct SGeom {
    static constexpr int kThreads = (B == 2048) ? BNBQ_STEP_THREADS_2048 : BNBQ_STEP_THREADS;
    static constexpr int G = B / kEPT;                 // threads per block-group
    static constexpr int kGroups = kThreads / G;       // block-groups per CTA
    static constexpr int kGroupWarps = G >= 32 ? G / 32 : 1;
    static_assert(kThreads % G == 0 && (G <= 32 || kGroups <= 15), "groups fit the CTA and the named barriers");
};

template <int OPT>
struct OptTraits {
    static constexpr bool kTwoStates = (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM);
    static constexpr int kCodes = kTwoStates ? 2 : 1;
};

// Scalars as pairs for the packed instructions.
struct Pairs {
    float2 b1, b2, omb1, omb2, decay, nstep, rcp_sqrt_bc2, nsqrt_bc2, eps, wd, nlr;
};

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

__device__ __forceinline__ Pairs make_pairs(const StepScalars& sc)
{
    Pairs q;
    q.b1 = f2(sc.b1); q.b2 = f2(sc.b2); q.omb1 = f2(sc.omb1); q.omb2 = f2(sc.omb2);
    q.decay = f2(sc.decay); q.nstep = f2(-sc.step_size); q.rcp_sqrt_bc2 = f2(sc.rcp_sqrt_bc2);
    q.nsqrt_bc2 = f2(-sc.sqrt_bc2); q.eps = f2(sc.eps); q.wd = f2(sc.wd); q.nlr = f2(-sc.lr);
    return q;
}

// The update of one pair of elements, in two parts.  Every binary32 operation is rounded on its
// own, in the order the header documents; p - c*u is formed as p + (-c)*u, which rounds
// identically.
//
// Part 1 (states2): the new optimizer states from the old ones and g.  Lion and momentum, whose
// parameter update needs no square root or division, also update p here.  Afterwards `m` and `v`
// hold what part 2 reads: AdamW/Adam m' and v'; RMSprop v' (its one state) and the gradient
// (with weight decay added) in `v`.
template <int OPT>
__device__ __forceinline__ void states2(const StepScalars& sc, const Pairs& k, float2& p, float2 g,
                                        float2& m, float2& v)
{
    if constexpr (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM) {
        if constexpr (OPT == BNBQ_ADAM) {
            if (sc.wd != 0.0f) g = add2(g, mul2(k.wd, p));
        }
        m = add2(mul2(k.b1, m), mul2(k.omb1, g));
        v = add2(mul2(k.b2, v), mul2(mul2(k.omb2, g), g));
    } else if constexpr (OPT == BNBQ_LION) {
        const float2 c = add2(mul2(k.b1, m), mul2(k.omb1, g));
        const float2 sg = make_float2((c.x > 0.0f) ? 1.0f : ((c.x < 0.0f) ? -1.0f : 0.0f),
                                      (c.y > 0.0f) ? 1.0f : ((c.y < 0.0f) ? -1.0f : 0.0f));
        p = mul2(p, k.decay);
        p = add2(p, mul2(k.nlr, sg));
        m = add2(mul2(k.b2, m), mul2(k.omb2, g));
    } else if constexpr (OPT == BNBQ_MOMENTUM) {  // dampening 0
        if (sc.wd != 0.0f) g = add2(g, mul2(k.wd, p));
        const float2 m1 = add2(mul2(k.b1, m), g);
        p = add2(p, mul2(k.nlr, m1));
        m = m1;
    } else {  // RMSprop: the one state (m) is the running mean of squares, b1 = alpha
        if (sc.wd != 0.0f) g = add2(g, mul2(k.wd, p));
        m = add2(mul2(k.b1, m), mul2(mul2(k.omb1, g), g));
        v = g;
    }
}

// Optimizers whose parameter update takes a square root and a division (part 2).
template <int OPT>
constexpr bool kHasPart2 = (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM || OPT == BNBQ_RMSPROP);

// Part 2: the parameter update from part 1's (m, v).  FAST takes the FMA square root and
// division, which are exact when the square root's operand lies in [kSqrtOpLo, kSqrtOpHi] and
// the numerator's magnitude in [kDivNumLo, kDivNumHi] (the caller checks; with those, the host's
// checks eps <= 2^60 and sqrt(1-b2^t) in [2^-12, 1] keep the denominator in [2^-50, 2^63] and the
// quotient's magnitude in [2^-123, 2^110]); otherwise the IEEE intrinsics.
// sqrt(v)/sqrt(1-b2^t) always uses the FMA quotient: the host rejects sqrt(1-b2^t) outside
// [2^-60, 1] (any binary32 b2 < 1 gives at least 2^-12), and sqrt(v) is 0 or at least 2^-75, so
// the quotient is the correctly rounded one.
template <int OPT, bool FAST>
__device__ __forceinline__ void p_update2(const Pairs& k, float2& p, float2 m, float2 v)
{
    if constexpr (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM) {
        if constexpr (OPT == BNBQ_ADAMW) p = mul2(p, k.decay);
        const float2 s = FAST ? sqrt2_ranged(v) : make_float2(__fsqrt_rn(v.x), __fsqrt_rn(v.y));
        const float2 den = add2(div2_rcp(s, k.rcp_sqrt_bc2, k.nsqrt_bc2), k.eps);
        const float2 u = FAST ? div2_ranged(m, den) : make_float2(__fdiv_rn(m.x, den.x), __fdiv_rn(m.y, den.y));
        p = add2(p, mul2(k.nstep, u));
    } else if constexpr (OPT == BNBQ_RMSPROP) {  // m = v', v = g
        const float2 s = FAST ? sqrt2_ranged(m) : make_float2(__fsqrt_rn(m.x), __fsqrt_rn(m.y));
        const float2 den = add2(s, k.eps);
        const float2 u = FAST ? div2_ranged(v, den) : make_float2(__fdiv_rn(v.x, den.x), __fdiv_rn(v.y, den.y));
        p = add2(p, mul2(k.nlr, u));
    }
}

// Both parts with the IEEE square root and division (32-bit state path).
template <int OPT>
__device__ __forceinline__ void update2(const StepScalars& sc, const Pairs& k, float2& p, float2 g,
                                        float2& m, float2& v)
{
    states2<OPT>(sc, k, p, g, m, v);
    if constexpr (kHasPart2<OPT>) p_update2<OPT, false>(k, p, m, v);
}

// Range test for the FAST part 2, from the extremes of the operands over the thread's elements
// (hi1/lo1: largest/smallest |m|, hi2/lo2: the same for v).
template <int OPT>
__device__ __forceinline__ bool part2_in_range(float hi1, float lo1, float hi2, float lo2)
{
    if constexpr (OPT == BNBQ_RMSPROP)  // m is the square root's operand, v the numerator
        return hi1 <= kSqrtOpHi && lo1 >= kSqrtOpLo && hi2 <= kDivNumHi && lo2 >= kDivNumLo;
    else
        return hi1 <= kDivNumHi && lo1 >= kDivNumLo && hi2 <= kSqrtOpHi && lo2 >= kSqrtOpLo;
}

// ---- codebook tables of the step kernel ---------------------------------------------------------
// Dequantizing the states looks up code[q] for random q: with one copy of the 256 codes, a warp's
// 32 lookups land in random banks and cost about 3.4 shared-memory wavefronts.  crep holds 32
// copies interleaved, code[q] at [32 q + b] for every bank b, and lane L reads copy L: each lane
// in its own bank, one wavefront per lookup (32 KB per codebook; measured 0.7-0.8% faster on the
// 7B list, at full clock and under the power limit).
// The bucket tables hold only the indices that a normalised value in [-1, 1] reaches: the signed
// table of the first state [kSignedLo, kSignedHi] and, for a second codebook without negative
// codes, the non-negative table [kNonNegLo, kSignedHi] (about 44 KB for both).  The padding
// around them keeps every index that any bit pattern can form ([-kHalf, kHalf) around each
// table's index 0) inside the allocation.  The footprint still leaves most of the SM's unified
// L1/shared memory to L1, where the streamed loads land while in flight.
constexpr int kCodeRep = 32;
template <int NC>
struct StepSmem {
    float crep[NC][256 * kCodeRep];  // code[q] at [q * kCodeRep + lane % kCodeRep]
    float code[NC][256];
    float mid[NC][256];
    uint32_t pad0[NC == 2 ? 4 : 260];
    uint32_t stab[kSignedHi - kSignedLo + 1];
    uint32_t utab[NC == 2 ? kSignedHi - kNonNegLo + 1 : 4];
    uint32_t pad1[128];

    __device__ __forceinline__ const uint32_t* center1() const { return stab - kSignedLo; }
    __device__ __forceinline__ const uint32_t* center2() const { return utab - kNonNegLo; }
};

// The second state's codebook has negative codes: binary search over its midpoints.
constexpr int kSearchBinary = 3;

template <int MODE>
__device__ __forceinline__ uint32_t step_code_word(const uint32_t* center, const float* mid, float x)
{
    if constexpr (MODE == kSearchBinary)
        return (uint32_t)count_mid_below(mid, 256, x) << 24;
    else
        return nearest_code_word<MODE>(center, mid, x);
}

// ---- guarded element access for the partial last block of a tensor -----------------------------
__device__ __forceinline__ float4 load_f4_guard(const float* p, int64_t e, int64_t n)
{
    if (e + 4 <= n) return ld_stream_f4(p + e);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e + 0 < n) v.x = p[e + 0];
    if (e + 1 < n) v.y = p[e + 1];
    if (e + 2 < n) v.z = p[e + 2];
    return v;
}

__device__ __forceinline__ void store_f4_guard(float* p, int64_t e, int64_t n, float4 v)
{
    if (e + 4 <= n) { st_stream_f4(p + e, v); return; }
    if (e + 0 < n) p[e + 0] = v.x;
    if (e + 1 < n) p[e + 1] = v.y;
    if (e + 2 < n) p[e + 2] = v.z;
}

__device__ __forceinline__ float4 load_g4(const void* g, bool bf16, int64_t e, int64_t n, bool full)
{
    if (full || e + 4 <= n) {
        if (bf16) {
            const uint2 w = ld_stream_u2(static_cast<const uint16_t*>(g) + e);
            return make_float4(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x), bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
        }
        return ld_stream_f4(static_cast<const float*>(g) + e);
    }
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < 3; i++)
        if (e + i < n)
            v[i] = bf16 ? __uint_as_float((uint32_t)(static_cast<const uint16_t*>(g)[e + i]) << 16)
                        : static_cast<const float*>(g)[e + i];
    return make_float4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ uint32_t load_q4(const uint8_t* q, int64_t e, int64_t n, bool full)
{
    if (full || e + 4 <= n) return ld_stream_u32(q + e);
    uint32_t w = 0;
    for (int i = 0; i < 3; i++)
        if (e + i < n) w |= (uint32_t)q[e + i] << (8 * i);
    return w;
}

__device__ __forceinline__ void store_q4(uint8_t* q, int64_t e, int64_t n, uint32_t w, bool full)
{
    if (full || e + 4 <= n) { st_stream_u32(q + e, w); return; }
    for (int i = 0; i < 3; i++)
        if (e + i < n) q[e + i] = (uint8_t)(w >> (8 * i));
}

__device__ __forceinline__ uint32_t byte_of(uint32_t w, int i) { return __byte_perm(w, 0u, 0x4440u + (uint32_t)i); }

// code[byte i of w] from the lane's copy in crep (`code` = crep + lane % kCodeRep), with the
// byte's offset 128 * byte formed by one shift and one mask (i is a compile-time constant in the
// unrolled loops).
static_assert(kCodeRep == 32, "code_at forms 4 * kCodeRep * byte as byte << 7");
__device__ __forceinline__ float code_at(const float* code, uint32_t w, int i)
{
    const uint32_t off = (i == 0 ? (w << 7) : (w >> (8 * i - 7))) & 0x7f80u;
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(code) + off);
}

// Group-wide max of (x, y) over the G threads of one block-group, in two halves so that work
// independent of the result can run between them: group_max_publish reduces inside each warp
// (and, for groups of several warps, stores the warp's maxima to shared memory, double-buffered
// by `parity`); group_max_collect waits at the group's named barrier and combines the warps.
template <int G, int NC>
__device__ __forceinline__ void group_max_publish(float& x, float& y, int gi, int tg, int lane, unsigned gmask,
                                                  float* red, int parity)
{
    if constexpr (G <= 32) {
        x = group_max_nan<G>(x, gmask);
        if constexpr (NC == 2) y = group_max_nan<G>(y, gmask);
    } else {
        constexpr int W = G / 32;
        x = group_max_nan<32>(x, 0xffffffffu);
        if constexpr (NC == 2) y = group_max_nan<32>(y, 0xffffffffu);
        float* r = red + ((gi * 2 + parity) * 2) * W;
        const int w = tg >> 5;
        if (lane == 0) {
            r[w] = x;
            if constexpr (NC == 2) r[W + w] = y;
        }
    }
}

template <int G, int NC>
__device__ __forceinline__ void group_max_collect(float& x, float& y, int gi, float* red, int& parity)
{
    if constexpr (G > 32) {
        constexpr int W = G / 32;
        const float* r = red + ((gi * 2 + parity) * 2) * W;
        group_barrier(1 + gi, G);
#pragma unroll
        for (int i = 0; i < W; i++) {
            x = max_nan(x, r[i]);
            if constexpr (NC == 2) y = max_nan(y, r[W + i]);
        }
        parity ^= 1;
    }
}

// The current tensor's descriptor, held in registers while a group walks its blocks.
struct Cur {
    float* p;
    const void* g;
    uint8_t* q1;
    uint8_t* q2;
    float* a1;
    float* a2;
    int64_t n;
    int first;
    int flags;
};

__device__ __forceinline__ void load_cur(Cur& c, const StepDesc* __restrict__ table, int i, int ntensors)
{
    const uint4* d = reinterpret_cast<const uint4*>(table + i);
    const uint4 w0 = __ldg(d), w1 = __ldg(d + 1), w2 = __ldg(d + 2), w3 = __ldg(d + 3);
    auto ptr = [](uint32_t lo, uint32_t hi) {
        return reinterpret_cast<void*>(((unsigned long long)hi << 32) | lo);
    };
    c.p = static_cast<float*>(ptr(w0.x, w0.y));
    c.g = ptr(w0.z, w0.w);
    c.q1 = static_cast<uint8_t*>(ptr(w1.x, w1.y));
    c.q2 = static_cast<uint8_t*>(ptr(w1.z, w1.w));
    c.a1 = static_cast<float*>(ptr(w2.x, w2.y));
    c.a2 = static_cast<float*>(ptr(w2.z, w2.w));
    c.n = (int64_t)(((unsigned long long)w3.y << 32) | w3.x);
    c.first = (int)w3.z;
    c.flags = (int)w3.w;
}

// Requantize the kNCH chunks of one block: FAST selects the FMA quotient; M1 / M2 are the
// search modes of the two codebooks.
template <int OPT, int B, bool FULL, int M1, int M2, bool FAST>
__device__ __forceinline__ void requant(const Cur& c, int64_t base, int tg, const StepSmem<OptTraits<OPT>::kCodes>& sm,
                                        const float2 (&mv)[2 * kNCH], const float2 (&vv)[2 * kNCH],
                                        const BlockScale& s1, const BlockScale& s2)
{
    constexpr int G = SGeom<B>::G;
    constexpr bool TWO = OptTraits<OPT>::kTwoStates;
    const float2 r1 = f2(s1.r), na1 = f2(s1.na), r2 = f2(s2.r), na2 = f2(s2.na);
    const uint32_t* t1 = sm.center1();
    const uint32_t* t2 = sm.center2();
    const float* mid1 = sm.mid[0];
    const float* mid2 = sm.mid[TWO ? 1 : 0];
#pragma unroll
    for (int j = 0; j < kNCH; j++) {
        const int64_t e = base + 4 * (j * G + tg);
        if (!FULL && e >= c.n) continue;
        uint32_t w1[4], w2[4];
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const float2 xn = FAST ? div2_rcp(mv[2 * j + h], r1, na1)
                                   : make_float2(__fdiv_rn(mv[2 * j + h].x, s1.a), __fdiv_rn(mv[2 * j + h].y, s1.a));
            w1[2 * h] = step_code_word<M1>(t1, mid1, xn.x);
            w1[2 * h + 1] = step_code_word<M1>(t1, mid1, xn.y);
            if constexpr (TWO) {
                const float2 yn = FAST ? div2_rcp(vv[2 * j + h], r2, na2)
                                       : make_float2(__fdiv_rn(vv[2 * j + h].x, s2.a), __fdiv_rn(vv[2 * j + h].y, s2.a));
                w2[2 * h] = step_code_word<M2>(t2, mid2, yn.x);
                w2[2 * h + 1] = step_code_word<M2>(t2, mid2, yn.y);
            }
        }
        store_q4(c.q1, e, c.n, pack_top_bytes(w1[0], w1[1], w1[2], w1[3]), FULL);
        if constexpr (TWO) store_q4(c.q2, e, c.n, pack_top_bytes(w2[0], w2[1], w2[2], w2[3]), FULL);
    }
}

// Gradient chunk held in its loaded form until the update needs it.
template <bool GB>
struct GRaw;
template <>
struct GRaw<true> {
    uint2 w;
    __device__ __forceinline__ float2 half(int h) const
    {
        const uint32_t x = h ? w.y : w.x;
        return make_float2(bf16lo_to_f32(x), bf16hi_to_f32(x));
    }
};
template <>
struct GRaw<false> {
    float4 f;
    __device__ __forceinline__ float2 half(int h) const { return h ? make_float2(f.z, f.w) : make_float2(f.x, f.y); }
};

template <bool GB, bool FULL>
__device__ __forceinline__ GRaw<GB> load_graw(const void* g, int64_t e, int64_t n)
{
    GRaw<GB> r;
    if constexpr (GB) {
        const uint16_t* gh = static_cast<const uint16_t*>(g);
        if (FULL || e + 4 <= n) {
            r.w = ld_stream_u2(gh + e);
        } else {
            uint32_t v[3] = {0u, 0u, 0u};
            for (int i = 0; i < 3; i++)
                if (e + i < n) v[i] = gh[e + i];
            r.w = make_uint2(v[0] | (v[1] << 16), v[2]);
        }
    } else {
        r.f = FULL ? ld_stream_f4(static_cast<const float*>(g) + e) : load_f4_guard(static_cast<const float*>(g), e, n);
    }
    return r;
}

// One block with 8-bit state.  FULL: the block lies entirely inside the tensor; GB: bf16 grads.
template <int OPT, int B, bool FULL, int M1, int M2, bool GB>
__device__ __forceinline__ void block8(const Cur& c, int64_t lb, const StepScalars& sc, const Pairs& kp,
                                       const StepSmem<OptTraits<OPT>::kCodes>& cs, bool fast1, bool fast2, int gi,
                                       int tg, int lane, unsigned gmask, float* red, int& parity, unsigned* flags)
{
    constexpr int G = SGeom<B>::G;
    constexpr bool TWO = OptTraits<OPT>::kTwoStates;
    constexpr int NC = OptTraits<OPT>::kCodes;
    constexpr bool P2 = kHasPart2<OPT>;
    const float* code1 = cs.crep[0] + (lane % kCodeRep);
    const float* code2 = cs.crep[NC - 1] + (lane % kCodeRep);
    const int64_t n = c.n;
    const int64_t base = lb * B;
    const int64_t e0 = base + 4 * tg;  // chunk j starts at e0 + 4*G*j

    // a4: loads
    float4 pv[kNCH];
    GRaw<GB> gv[kNCH];
    uint32_t w1[kNCH], w2[kNCH];
#pragma unroll
    for (int j = 0; j < kNCH; j++) {
        const int64_t e = e0 + 4 * G * j;
        pv[j] = FULL ? ld_stream_f4(c.p + e) : load_f4_guard(c.p, e, n);
        gv[j] = load_graw<GB, FULL>(c.g, e, n);
        w1[j] = load_q4(c.q1, e, n, FULL);
        if constexpr (TWO) w2[j] = load_q4(c.q2, e, n, FULL);
    }
    const float a1 = __ldg(c.a1 + lb);
    const float a2 = TWO ? __ldg(c.a2 + lb) : 0.0f;
    const float2 a1p = f2(a1), a2p = f2(a2);

    // a4 + a5: dequantize, new states, parameter update; store p
    float2 mv[2 * kNCH], vv[2 * kNCH];
    float mx1 = 0.0f, mx2 = 0.0f;  // block absmax partials
    // Running extremes of part 2's operands (|m|, |v|) over the thread's chunks so far: part 2 of a
    // chunk takes the FMA square root and division when they lie in the exact range for every
    // thread of the warp (one warp-uniform choice per chunk).
    float lo1 = __int_as_float(0x7f800000), lo2 = lo1, hi2 = 0.0f;
#pragma unroll
    for (int j = 0; j < kNCH; j++) {
        const int64_t e = e0 + 4 * G * j;
        float2 ph[2] = {make_float2(pv[j].x, pv[j].y), make_float2(pv[j].z, pv[j].w)};
#pragma unroll
        for (int h = 0; h < 2; h++) {
            float2 m = mul2(make_float2(code_at(code1, w1[j], 2 * h), code_at(code1, w1[j], 2 * h + 1)), a1p);
            float2 v = make_float2(0.0f, 0.0f);
            if constexpr (TWO)
                v = mul2(make_float2(code_at(code2, w2[j], 2 * h), code_at(code2, w2[j], 2 * h + 1)), a2p);
            states2<OPT>(sc, kp, ph[h], gv[j].half(h), m, v);
            if (!FULL) {  // elements past the end do not count towards the block scale
                if (e + 2 * h >= n) { m.x = 0.0f; v.x = 0.0f; }
                if (e + 2 * h + 1 >= n) { m.y = 0.0f; v.y = 0.0f; }
            }
            mv[2 * j + h] = m;
            vv[2 * j + h] = v;
            mx1 = max3_abs_nan(mx1, m.x, m.y);
            if constexpr (TWO) mx2 = max3_abs_nan(mx2, v.x, v.y);
            if constexpr (P2 && FULL) {
                lo1 = min3_abs(lo1, m.x, m.y);
                lo2 = min3_abs(lo2, v.x, v.y);
                if constexpr (!TWO) hi2 = max3_abs_nan(hi2, v.x, v.y);
            }
        }
        if constexpr (P2) {
            bool fast = false;
            if constexpr (FULL)
                fast = __all_sync(gmask, sc.upd_fast && part2_in_range<OPT>(mx1, lo1, TWO ? mx2 : hi2, lo2));
            if (fast) {
                p_update2<OPT, true>(kp, ph[0], mv[2 * j], vv[2 * j]);
                p_update2<OPT, true>(kp, ph[1], mv[2 * j + 1], vv[2 * j + 1]);
            } else {
                p_update2<OPT, false>(kp, ph[0], mv[2 * j], vv[2 * j]);
                p_update2<OPT, false>(kp, ph[1], mv[2 * j + 1], vv[2 * j + 1]);
            }
        }
        const float4 po = make_float4(ph[0].x, ph[0].y, ph[1].x, ph[1].y);
        if (FULL) {
            st_stream_f4(c.p + e, po);
        } else if (e < n) {
            store_f4_guard(c.p, e, n, po);
        }
    }

    // a6: block absmax of the new states
    float r1 = mx1, r2 = mx2;
    group_max_publish<G, NC>(r1, r2, gi, tg, lane, gmask, red, parity);
    group_max_collect<G, NC>(r1, r2, gi, red, parity);
    if (tg == 0) {
        c.a1[lb] = r1;
        if constexpr (TWO) c.a2[lb] = r2;
        if (!(r1 <= FLT_MAX) || !(r2 <= FLT_MAX)) atomicOr(flags, kFlagNonFinite);
    }

    // a7: requantize (one block-uniform choice of quotient)
    const BlockScale s1 = make_scale(r1, fast1);
    const BlockScale s2 = TWO ? make_scale(r2, fast2) : s1;
    if (s1.fast && s2.fast)
        requant<OPT, B, FULL, M1, M2, true>(c, base, tg, cs, mv, vv, s1, s2);
    else
        requant<OPT, B, FULL, M1, M2, false>(c, base, tg, cs, mv, vv, s1, s2);
}

// One block with 32-bit state (no quantization).
template <int OPT, int B>
__device__ __forceinline__ void block32(const Cur& c, int64_t lb, const StepScalars& sc, const Pairs& kp, int tg,
                                        unsigned gmask)
{
    constexpr int G = SGeom<B>::G;
    constexpr bool TWO = OptTraits<OPT>::kTwoStates;
    const int64_t n = c.n;
    const int64_t base = lb * B;
    float* m32 = reinterpret_cast<float*>(c.q1);
    float* v32 = reinterpret_cast<float*>(c.q2);
    const bool gbf16 = (c.flags & kDescGBf16) != 0;
    const bool full = base + B <= n;
#pragma unroll
    for (int j = 0; j < kNCH; j++) {
        const int64_t e = base + 4 * (j * G + tg);
        if (e >= n) continue;
        const float4 pv = load_f4_guard(c.p, e, n);
        const float4 gv = load_g4(c.g, gbf16, e, n, full);
        const float4 mq = load_f4_guard(m32, e, n);
        const float4 vq = TWO ? load_f4_guard(v32, e, n) : make_float4(0.f, 0.f, 0.f, 0.f);
        float2 ph[2] = {make_float2(pv.x, pv.y), make_float2(pv.z, pv.w)};
        float2 mh[2] = {make_float2(mq.x, mq.y), make_float2(mq.z, mq.w)};
        float2 vh[2] = {make_float2(vq.x, vq.y), make_float2(vq.z, vq.w)};
        states2<OPT>(sc, kp, ph[0], make_float2(gv.x, gv.y), mh[0], vh[0]);
        states2<OPT>(sc, kp, ph[1], make_float2(gv.z, gv.w), mh[1], vh[1]);
        if constexpr (kHasPart2<OPT>) {
            // FMA square root and division when the chunk's operands lie in their exact range for
            // the whole warp (full blocks only, where every thread of the group takes this chunk)
            bool fast = false;
            if (full) {
                const float hi1 = max_nan(max_nan(fabsf(mh[0].x), fabsf(mh[0].y)), max_nan(fabsf(mh[1].x), fabsf(mh[1].y)));
                const float lo1 = fminf(fminf(fabsf(mh[0].x), fabsf(mh[0].y)), fminf(fabsf(mh[1].x), fabsf(mh[1].y)));
                const float hi2 = max_nan(max_nan(fabsf(vh[0].x), fabsf(vh[0].y)), max_nan(fabsf(vh[1].x), fabsf(vh[1].y)));
                const float lo2 = fminf(fminf(fabsf(vh[0].x), fabsf(vh[0].y)), fminf(fabsf(vh[1].x), fabsf(vh[1].y)));
                fast = __all_sync(gmask, sc.upd_fast && part2_in_range<OPT>(hi1, lo1, hi2, lo2));
            }
            if (fast) {
                p_update2<OPT, true>(kp, ph[0], mh[0], vh[0]);
                p_update2<OPT, true>(kp, ph[1], mh[1], vh[1]);
            } else {
                p_update2<OPT, false>(kp, ph[0], mh[0], vh[0]);
                p_update2<OPT, false>(kp, ph[1], mh[1], vh[1]);
            }
        }
        store_f4_guard(c.p, e, n, make_float4(ph[0].x, ph[0].y, ph[1].x, ph[1].y));
        store_f4_guard(m32, e, n, make_float4(mh[0].x, mh[0].y, mh[1].x, mh[1].y));
        if constexpr (TWO) store_f4_guard(v32, e, n, make_float4(vh[0].x, vh[0].y, vh[1].x, vh[1].y));
    }
}

template <int OPT, int B, int M1, int M2>
__device__ __forceinline__ void step_loop(const StepDesc* __restrict__ table, int ntensors, int total_blocks,
                                          const StepScalars& sc, const StepSmem<OptTraits<OPT>::kCodes>& cs,
                                          bool fast1, bool fast2, float* red, unsigned* flags)
{
    using Geo = SGeom<B>;
    constexpr int G = Geo::G;
    const Pairs kp = make_pairs(sc);
    const int gi = threadIdx.x / G;
    const int tg = threadIdx.x % G;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G >= 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
    int parity = 0;
    int cur = -1;
    int next_first = 0;  // first block of tensor cur + 1 (INT_MAX past the last tensor)
    for (int b = blockIdx.x * Geo::kGroups + gi; b < total_blocks; b += gridDim.x * Geo::kGroups) {
        while (b >= next_first) {  // this block starts a later tensor: advance the cursor
            cur++;
            next_first = cur + 1 < ntensors ? __ldg(&table[cur + 1].first_block) : INT_MAX;
        }
        // The descriptor is re-read for every block (four 16-byte loads, L1-resident) rather than
        // kept in registers across blocks, which the update needs.
        Cur c;
        load_cur(c, table, cur, ntensors);
        const int64_t lb = (int64_t)(b - c.first);
        if (c.flags & kDescState8) {
            const bool full = (lb + 1) * B <= c.n;
            if (c.flags & kDescGBf16) {
                if (full)
                    block8<OPT, B, true, M1, M2, true>(c, lb, sc, kp, cs, fast1, fast2, gi, tg, lane, gmask, red, parity, flags);
                else
                    block8<OPT, B, false, M1, M2, true>(c, lb, sc, kp, cs, fast1, fast2, gi, tg, lane, gmask, red, parity, flags);
            } else {
                if (full)
                    block8<OPT, B, true, M1, M2, false>(c, lb, sc, kp, cs, fast1, fast2, gi, tg, lane, gmask, red, parity, flags);
                else
                    block8<OPT, B, false, M1, M2, false>(c, lb, sc, kp, cs, fast1, fast2, gi, tg, lane, gmask, red, parity, flags);
            }
        } else {
            block32<OPT, B>(c, lb, sc, kp, tg, gmask);
        }
    }
}

template <int OPT, int B>
__global__ void __launch_bounds__(SGeom<B>::kThreads, BNBQ_STEP_MIN_CTAS)
step_kernel(const StepDesc* __restrict__ table, int ntensors, int total_blocks, const StepScalars sc,
            const float* __restrict__ code1, const float* __restrict__ code2, unsigned* flags)
{
    constexpr int NC = OptTraits<OPT>::kCodes;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StepSmem<NC>& cs = *reinterpret_cast<StepSmem<NC>*>(smem_raw);
    float* red = reinterpret_cast<float*>(smem_raw + sizeof(StepSmem<NC>));

    // a0: codebook stage (skipped when the list has no 8-bit tensor)
    bool fast1 = true, fast2 = true, general = false, nonneg2 = true;
    if (code1 != nullptr) {
        stage_codes(cs.code[0], code1, 256);
        if constexpr (NC == 2) stage_codes(cs.code[1], code2, 256);
        __syncthreads();
        for (int k = threadIdx.x; k < 256 * kCodeRep; k += blockDim.x) {
            cs.crep[0][k] = cs.code[0][k / kCodeRep];
            if constexpr (NC == 2) cs.crep[NC - 1][k] = cs.code[NC - 1][k / kCodeRep];
        }
        bool bad = false, t1 = false, t2 = false;
        stage_midpoints(cs.code[0], cs.mid[0], 256, bad, t1);
        if constexpr (NC == 2) stage_midpoints(cs.code[1], cs.mid[1], 256, bad, t2);
        bad = __syncthreads_or(bad);
        fast1 = !__syncthreads_or(t1);
        fast2 = !__syncthreads_or(t2);
        if (bad) {
            if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(flags, kFlagBadCode);
            return;
        }
        nonneg2 = NC == 1 || cs.code[NC - 1][0] >= 0.0f;  // every code of the second state >= 0
        bool gen = build_bucket_entries(cs.stab - kSignedLo, cs.mid[0], 256, kSignedLo, kSignedHi);
        if (NC == 2 && nonneg2) gen |= build_bucket_entries(cs.utab - kNonNegLo, cs.mid[NC - 1], 256, kNonNegLo, kSignedHi);
        general = __syncthreads_or(gen);
    }
    if (!nonneg2)
        step_loop<OPT, B, kSearchGeneral, kSearchBinary>(table, ntensors, total_blocks, sc, cs, fast1, fast2, red, flags);
    else if (general)
        step_loop<OPT, B, kSearchGeneral, kSearchGeneral>(table, ntensors, total_blocks, sc, cs, fast1, fast2, red, flags);
    else
        step_loop<OPT, B, kSearchSigned, kSearchNonNeg>(table, ntensors, total_blocks, sc, cs, fast1, fast2, red, flags);
}

template <int OPT, int B>
constexpr size_t step_smem_bytes()
{
    return sizeof(StepSmem<OptTraits<OPT>::kCodes>) +
           sizeof(float) * SGeom<B>::kGroups * 2 * 2 * SGeom<B>::kGroupWarps;
}

template <int OPT, int B>
bnbq_status launch_step_t(const StepDesc* d_table, int ntensors, int total_blocks, const StepScalars& sc,
                          const float* code1, const float* code2, cudaStream_t s)
{
    using Geo = SGeom<B>;
    unsigned* flags = nullptr;
    bnbq_status st = device_flag_ptr(&flags);
    if (st != BNBQ_OK) return st;
    auto kern = step_kernel<OPT, B>;
    constexpr size_t smem = step_smem_bytes<OPT, B>();
    // The kernel's shared-memory limit and its resident CTAs per SM, set up once per device (for
    // this optimizer and blocksize) by whichever call first launches it there.
    constexpr int kDevs = 64;
    static std::mutex mu;
    static int per_sm_of[kDevs] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kDevs) return fail(BNBQ_EUNSUPPORTED, "device ordinal %d", dev);
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!per_sm_of[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(step smem)");
            int v = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, Geo::kThreads, smem);
            if (e != cudaSuccess) return cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
            if (v < 1) return fail(BNBQ_ECUDA, "step kernel does not fit on an SM");
            per_sm_of[dev] = v;
        }
        per_sm = per_sm_of[dev];
    }
    int sms = 0;
    st = sm_count(&sms);
    if (st != BNBQ_OK) return st;
    const int64_t need = ((int64_t)total_blocks + Geo::kGroups - 1) / Geo::kGroups;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    kern<<<grid, Geo::kThreads, smem, s>>>(d_table, ntensors, total_blocks, sc, code1, code2, flags);
    return cuda_status(cudaGetLastError(), "step_kernel launch");
}

template <int OPT>
bnbq_status launch_step_o(const StepDesc* t, int nt, int tb, const StepScalars& sc, const float* c1,
                          const float* c2, int B, cudaStream_t s)
{
    switch (B) {
        case 256: return launch_step_t<OPT, 256>(t, nt, tb, sc, c1, c2, s);
        case 2048: return launch_step_t<OPT, 2048>(t, nt, tb, sc, c1, c2, s);
        case 4096: return launch_step_t<OPT, 4096>(t, nt, tb, sc, c1, c2, s);
        default: return fail(BNBQ_EINVAL, "blocksize %d not in {256, 2048, 4096}", B);
    }
}

}  // namespace

bnbq_status launch_step(bnbq_optim opt, const StepDesc* d_table, int ntensors, int total_blocks,
                        const StepScalars& sc, const float* code1, const float* code2, int B,
                        cudaStream_t s)
{
    switch (opt) {
        case BNBQ_ADAMW: return launch_step_o<BNBQ_ADAMW>(d_table, ntensors, total_blocks, sc, code1, code2, B, s);
        case BNBQ_ADAM: return launch_step_o<BNBQ_ADAM>(d_table, ntensors, total_blocks, sc, code1, code2, B, s);
        case BNBQ_LION: return launch_step_o<BNBQ_LION>(d_table, ntensors, total_blocks, sc, code1, code2, B, s);
        case BNBQ_MOMENTUM: return launch_step_o<BNBQ_MOMENTUM>(d_table, ntensors, total_blocks, sc, code1, code2, B, s);
        case BNBQ_RMSPROP: return launch_step_o<BNBQ_RMSPROP>(d_table, ntensors, total_blocks, sc, code1, code2, B, s);
        default: return fail(BNBQ_EINVAL, "unknown optimizer %d", (int)opt);
    }
}

}  // namespace bnbq
