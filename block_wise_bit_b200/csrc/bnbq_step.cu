// bnbq_step.cu -- the fused multi-tensor 8-bit optimizer step for sm_100a.
//
// Method ("8-bit Optimizers via Block-wise Quantization", abstract, quoted on the blog.csdn.net
// bitsandbytes guide, section 2): optimizer statistics are kept in 8 bits with block-wise
// dynamic quantization while the update runs at 32-bit precision.  Per block this kernel
//   loads p (fp32), g (fp32/bf16), the 8-bit codes and the two block scales,
//   dequantizes m = code1[q1]*a1 and v = code2[q2]*a2 (codebooks staged in shared memory),
//   applies the fp32 AdamW / Adam / Lion / momentum update and stores p at once,
//   reduces the new block absmax of each state across the block's thread group,
//   requantizes each state against its new absmax (nearest code) and stores codes and scales.
// Tensors that keep 32-bit state (fewer than 4096 elements, and embedding tables: page
// "Py之bitsandbytes…详细攻略", section "如果需要高精度的参数") are stepped by the same launch.
//
// Scheduling: one launch per step for the whole tensor list.  The host uploads a table of
// tensor descriptors (cached across steps); blocks are numbered globally, tensor by tensor, and
// a persistent grid of SMs x resident CTAs strides over them.  Each block-group walks the
// table with a monotone cursor, so finding a block's tensor costs nothing per element.
//
// Roofline: HBM.  AdamW with 8-bit state and bf16 gradients moves 14 bytes per element
// (p read+write 8, g 2, q1 and q2 read+write 4) plus 16 bytes per block of scales.
#include <float.h>

#include "bnbq_device.cuh"
#include "bnbq_internal.h"

namespace bnbq {
namespace {

constexpr int kEPT = 16;

template <int B>
struct SGeom {
    static constexpr int G = B / kEPT;
    static constexpr int kThreads = G < 128 ? 128 : G;
    static constexpr int kGroups = kThreads / G;
    static constexpr int kWarps = kThreads / 32;
};

template <int OPT>
struct OptTraits {
    static constexpr bool kTwoStates = (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM);
};

// One element of the update.  Every binary32 operation is rounded on its own (explicit _rn
// intrinsics, never contracted), in the order the header documents.
template <int OPT>
__device__ __forceinline__ void update(const StepScalars& sc, float& p, float g, float& m, float& v)
{
    if constexpr (OPT == BNBQ_ADAMW || OPT == BNBQ_ADAM) {
        if constexpr (OPT == BNBQ_ADAM) {
            if (sc.wd != 0.0f) g = __fadd_rn(g, __fmul_rn(sc.wd, p));
        }
        const float m1 = __fadd_rn(__fmul_rn(sc.b1, m), __fmul_rn(sc.omb1, g));
        const float v1 = __fadd_rn(__fmul_rn(sc.b2, v), __fmul_rn(__fmul_rn(sc.omb2, g), g));
        if constexpr (OPT == BNBQ_ADAMW) p = __fmul_rn(p, sc.decay);
        const float s = __fsqrt_rn(v1);
        const float sn = sc.bc2_fast ? div_markstein(s, sc.sqrt_bc2, sc.rcp_sqrt_bc2)
                                     : __fdiv_rn(s, sc.sqrt_bc2);
        const float den = __fadd_rn(sn, sc.eps);
        p = __fsub_rn(p, __fmul_rn(sc.step_size, __fdiv_rn(m1, den)));
        m = m1;
        v = v1;
    } else if constexpr (OPT == BNBQ_LION) {
        const float c = __fadd_rn(__fmul_rn(sc.b1, m), __fmul_rn(sc.omb1, g));
        const float sg = (c > 0.0f) ? 1.0f : ((c < 0.0f) ? -1.0f : 0.0f);
        p = __fmul_rn(p, sc.decay);
        p = __fsub_rn(p, __fmul_rn(sc.lr, sg));
        m = __fadd_rn(__fmul_rn(sc.b2, m), __fmul_rn(sc.omb2, g));
    } else {  // momentum SGD, dampening 0
        if (sc.wd != 0.0f) g = __fadd_rn(g, __fmul_rn(sc.wd, p));
        const float m1 = __fadd_rn(__fmul_rn(sc.b1, m), g);
        p = __fsub_rn(p, __fmul_rn(sc.lr, m1));
        m = m1;
    }
}

__device__ __forceinline__ void load_p(const float* p, int64_t e, int64_t n, float (&v)[4])
{
    if (e + 4 <= n) {
        float4 f = ld_stream_f4(p + e);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++) v[i] = (e + i < n) ? p[e + i] : 0.0f;
    }
}

__device__ __forceinline__ void store_p(float* p, int64_t e, int64_t n, const float (&v)[4])
{
    if (e + 4 <= n) {
        st_stream_f4(p + e, make_float4(v[0], v[1], v[2], v[3]));
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++)
            if (e + i < n) p[e + i] = v[i];
    }
}

__device__ __forceinline__ void load_g(const void* g, bool bf16, int64_t e, int64_t n, float (&v)[4])
{
    if (e + 4 <= n) {
        if (bf16) {
            uint2 w = ld_stream_u2(static_cast<const uint16_t*>(g) + e);
            v[0] = bf16lo_to_f32(w.x); v[1] = bf16hi_to_f32(w.x);
            v[2] = bf16lo_to_f32(w.y); v[3] = bf16hi_to_f32(w.y);
        } else {
            float4 f = ld_stream_f4(static_cast<const float*>(g) + e);
            v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float x = 0.0f;
            if (e + i < n)
                x = bf16 ? __uint_as_float((uint32_t)(static_cast<const uint16_t*>(g)[e + i]) << 16)
                         : static_cast<const float*>(g)[e + i];
            v[i] = x;
        }
    }
}

__device__ __forceinline__ uint32_t load_q(const uint8_t* q, int64_t e, int64_t n)
{
    if (e + 4 <= n) return ld_stream_u32(q + e);
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; i++)
        if (e + i < n) w |= (uint32_t)q[e + i] << (8 * i);
    return w;
}

__device__ __forceinline__ void store_q(uint8_t* q, int64_t e, int64_t n, uint32_t w)
{
    if (e + 4 <= n) {
        st_stream_u32(q + e, w);
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++)
            if (e + i < n) q[e + i] = (uint8_t)(w >> (8 * i));
    }
}

template <int OPT, int B>
__global__ void __launch_bounds__(SGeom<B>::kThreads)
step_kernel(const StepDesc* __restrict__ table, int ntensors, int total_blocks, const StepScalars sc,
            const float* __restrict__ code1, const float* __restrict__ code2, unsigned* flags)
{
    using Geo = SGeom<B>;
    constexpr int G = Geo::G;
    constexpr bool TWO = OptTraits<OPT>::kTwoStates;
    constexpr int NCODE = TWO ? 2 : 1;
    __shared__ CodeSmem cs[NCODE];
    __shared__ float red[2][NCODE][Geo::kWarps];

    // a0: codebook stage (skipped when the list has no 8-bit tensor).
    bool tiny[NCODE];
    for (int c = 0; c < NCODE; c++) tiny[c] = false;
    if (code1 != nullptr) {
        stage_code_pass1(cs[0], code1, 256);
        if constexpr (TWO) stage_code_pass1(cs[1], code2, 256);
        __syncthreads();
        bool bad = false, t0 = false, t1 = false;
        stage_code_pass2(cs[0], 256, bad, t0);
        if constexpr (TWO) stage_code_pass2(cs[1], 256, bad, t1);
        bad = __syncthreads_or(bad);
        tiny[0] = __syncthreads_or(t0);
        if constexpr (TWO) tiny[NCODE - 1] = __syncthreads_or(t1);
        if (bad) {
            if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(flags, kFlagBadCode);
            return;
        }
        stage_code_pass3(cs[0], 256);
        if constexpr (TWO) stage_code_pass3(cs[1], 256);
        __syncthreads();
    }

    const int gi = threadIdx.x / G;
    const int tg = threadIdx.x % G;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const unsigned gmask = (G >= 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
    int parity = 0;
    int cur = 0;

    for (int b = blockIdx.x * Geo::kGroups + gi; b < total_blocks; b += gridDim.x * Geo::kGroups) {
        while (cur + 1 < ntensors && __ldg(&table[cur + 1].first_block) <= b) cur++;
        const StepDesc* d = table + cur;
        float* p = d->p;
        const void* gp = d->g;
        const int64_t n = d->n;
        const int dflags = d->flags;
        const bool gbf16 = (dflags & kDescGBf16) != 0;
        const int64_t lb = (int64_t)(b - d->first_block);
        const int64_t base = lb * B;

        if (dflags & kDescState8) {
            // a4: load + dequantize
            uint8_t* q1p = static_cast<uint8_t*>(d->s1);
            uint8_t* q2p = static_cast<uint8_t*>(d->s2);
            float pv[4][4], gv[4][4], mv[4][4], vv[4][4];
            uint32_t w1[4], w2[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int64_t e = base + 4 * (j * G + tg);
                load_p(p, e, n, pv[j]);
                load_g(gp, gbf16, e, n, gv[j]);
                w1[j] = load_q(q1p, e, n);
                if constexpr (TWO) w2[j] = load_q(q2p, e, n);
            }
            const float a1 = __ldg(d->a1 + lb);
            float a2 = 0.0f;
            if constexpr (TWO) a2 = __ldg(d->a2 + lb);

            // a5: update; p is stored at once
            float mx1 = 0.0f, mx2 = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int64_t e = base + 4 * (j * G + tg);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    float m = __fmul_rn(cs[0].code[(w1[j] >> (8 * i)) & 0xff], a1);
                    float v = 0.0f;
                    if constexpr (TWO) v = __fmul_rn(cs[NCODE - 1].code[(w2[j] >> (8 * i)) & 0xff], a2);
                    update<OPT>(sc, pv[j][i], gv[j][i], m, v);
                    if (e + i >= n) { m = 0.0f; v = 0.0f; }
                    mv[j][i] = m;
                    vv[j][i] = v;
                    mx1 = max_nan(mx1, fabsf(m));
                    if constexpr (TWO) mx2 = max_nan(mx2, fabsf(v));
                }
                if (e < n) store_p(p, e, n, pv[j]);
            }

            // a6: new block absmax of each state
            if constexpr (G <= 32) {
                mx1 = group_max_nan<G>(mx1, gmask);
                if constexpr (TWO) mx2 = group_max_nan<G>(mx2, gmask);
            } else {
                mx1 = group_max_nan<32>(mx1, 0xffffffffu);
                if constexpr (TWO) mx2 = group_max_nan<32>(mx2, 0xffffffffu);
                if (lane == 0) {
                    red[parity][0][warp] = mx1;
                    if constexpr (TWO) red[parity][NCODE - 1][warp] = mx2;
                }
                __syncthreads();
#pragma unroll
                for (int w = 0; w < Geo::kWarps; w++) {
                    mx1 = max_nan(mx1, red[parity][0][w]);
                    if constexpr (TWO) mx2 = max_nan(mx2, red[parity][NCODE - 1][w]);
                }
                parity ^= 1;
            }
            if (tg == 0) {
                d->a1[lb] = mx1;
                if constexpr (TWO) d->a2[lb] = mx2;
                if (!(mx1 <= FLT_MAX) || !(mx2 <= FLT_MAX)) atomicOr(flags, kFlagNonFinite);
            }

            // a7: requantize
            const BlockScale s1 = make_scale(mx1, !tiny[0]);
            BlockScale s2 = s1;
            if constexpr (TWO) s2 = make_scale(mx2, !tiny[NCODE - 1]);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int64_t e = base + 4 * (j * G + tg);
                if (e >= n) continue;
                uint32_t o1 = 0, o2 = 0;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    o1 |= nearest_code(cs[0], normalise(mv[j][i], s1)) << (8 * i);
                    if constexpr (TWO) o2 |= nearest_code(cs[NCODE - 1], normalise(vv[j][i], s2)) << (8 * i);
                }
                store_q(q1p, e, n, o1);
                if constexpr (TWO) store_q(q2p, e, n, o2);
            }
        } else {
            // a8: 32-bit state path (same update, no quantization)
            float* m32 = static_cast<float*>(d->s1);
            float* v32 = static_cast<float*>(d->s2);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int64_t e = base + 4 * (j * G + tg);
                if (e >= n) continue;
                float pv[4], gv[4], mv[4], vv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                load_p(p, e, n, pv);
                load_g(gp, gbf16, e, n, gv);
                load_p(m32, e, n, mv);
                if constexpr (TWO) load_p(v32, e, n, vv);
#pragma unroll
                for (int i = 0; i < 4; i++) update<OPT>(sc, pv[i], gv[i], mv[i], vv[i]);
                store_p(p, e, n, pv);
                store_p(m32, e, n, mv);
                if constexpr (TWO) store_p(v32, e, n, vv);
            }
        }
    }
}

template <int OPT, int B>
bnbq_status launch_step_t(const StepDesc* d_table, int ntensors, int total_blocks,
                          const StepScalars& sc, const float* code1, const float* code2,
                          cudaStream_t s)
{
    using Geo = SGeom<B>;
    unsigned* flags = nullptr;
    bnbq_status st = device_flag_ptr(&flags);
    if (st != BNBQ_OK) return st;
    auto kern = step_kernel<OPT, B>;
    static thread_local int cached_dev = -1, cached_per_sm = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (cached_dev != dev) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&cached_per_sm, kern, Geo::kThreads, 0);
        if (e != cudaSuccess) return cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        if (cached_per_sm < 1) cached_per_sm = 1;
        cached_dev = dev;
    }
    int sms = 0;
    st = sm_count(&sms);
    if (st != BNBQ_OK) return st;
    const int64_t need = ((int64_t)total_blocks + Geo::kGroups - 1) / Geo::kGroups;
    const int64_t cap = (int64_t)sms * cached_per_sm;
    const int grid = (int)(need < cap ? need : cap);
    kern<<<grid, Geo::kThreads, 0, s>>>(d_table, ntensors, total_blocks, sc, code1, code2, flags);
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
        default: return fail(BNBQ_EINVAL, "unknown optimizer %d", (int)opt);
    }
}

}  // namespace bnbq
