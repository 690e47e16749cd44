// bnbq_noalloc.cu -- bnbq_step_8bit_noalloc: the fused multi-tensor optimizer step for callers
// that cannot allocate device memory.
//
// bnbq_step_8bit keeps the per-list descriptor table in device memory it allocates itself (and
// caches).  Some callers cannot let a library call cudaMalloc: code running inside a memory
// pool or arena that owns all device memory, a process that must not grow its footprint after
// start-up, or a host loop that must never hit an allocator (and its implicit synchronisation)
// between steps.  This entry point runs the same step kernel, but its descriptor table lives in
// a fixed array compiled into the library (g_noalloc_table below, kNoAllocMaxTensors entries of
// 64 bytes = 256 KiB, held by every GPU that loads the library until the process exits).  It
// calls no cudaMalloc, cudaFree, cudaMallocHost or any allocating library routine.
//
// Set-up: the array's name is only a host-side stand-in for the device object, so its device
// address is looked up with cudaGetSymbolAddress once per device (with that device current),
// on the first call made on that device.  With CUDA's lazy module loading that first lookup may
// also load the library's device code onto the device, which is when the 256 KiB table (and
// the code) take device memory; the step kernel's shared-memory limit is likewise set up at the
// first step call on a device for each optimizer and blocksize.  A caller that must not allocate
// later should therefore make one call at start-up on each device it uses, and make it before
// capturing any stream.
//
// Sharing: every call on a device writes its table into the same array, which keeps the last
// call's contents.  Two calls whose work overlaps on the GPU (different streams, no ordering
// between them) race on the table; order them (same stream, or events) if you issue several.
// The table is fully rewritten for the entries a call uses, so nothing needs clearing.
#include <math.h>
#include <mutex>
#include <string.h>

#include "bnbq_internal.h"

namespace bnbq {
namespace {

constexpr int kNoAllocMaxTensors = 4096;  // non-empty tensors per call
constexpr int kNoAllocMaxDevices = 64;

// The step's scratch: one descriptor table per device, in the library's own device image.
static __device__ __align__(256) StepDesc g_noalloc_table[kNoAllocMaxTensors];

std::mutex g_na_mu;                           // guards the two arrays below
StepDesc* g_na_ptr[kNoAllocMaxDevices] = {};  // device address of g_noalloc_table, per device
StepDesc g_na_host[kNoAllocMaxTensors];       // host staging of the table (static storage)

bool aligned_na(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Device address of the table on the current device (looked up once per device); caller holds g_na_mu.
bnbq_status table_address(StepDesc** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(BNBQ_EUNSUPPORTED, "device ordinal %d", dev);
    if (!g_na_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_table);
        if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(step descriptor table)");
        g_na_ptr[dev] = static_cast<StepDesc*>(p);
    }
    *out = g_na_ptr[dev];
    return BNBQ_OK;
}

}  // namespace
}  // namespace bnbq

using namespace bnbq;

extern "C" BNBQ_API bnbq_status bnbq_step_8bit_noalloc(bnbq_optim opt, const bnbq_tensor* list, int ntensors,
                                                       const bnbq_hparams* hp, int step, const float* code1,
                                                       const float* code2, int blocksize, bnbq_stream_t stream)
{
    if (opt < BNBQ_ADAMW || opt > BNBQ_RMSPROP) return fail(BNBQ_EINVAL, "unknown optimizer %d", (int)opt);
    if (ntensors < 0) return fail(BNBQ_EINVAL, "ntensors %d < 0", ntensors);
    if (ntensors > 0 && !list) return fail(BNBQ_EINVAL, "list is NULL");
    if (!hp) return fail(BNBQ_EINVAL, "hp is NULL");
    if (step < 1) return fail(BNBQ_EINVAL, "step %d < 1", step);
    if (blocksize != 256 && blocksize != 2048 && blocksize != 4096)
        return fail(BNBQ_EINVAL, "blocksize %d not in {256, 2048, 4096}", blocksize);
    const float hv[5] = {hp->lr, hp->beta1, hp->beta2, hp->eps, hp->weight_decay};
    for (float x : hv)
        if (!isfinite(x)) return fail(BNBQ_EINVAL, "hyper-parameters must be finite");
    const bool two = (opt == BNBQ_ADAMW || opt == BNBQ_ADAM);
    if (two && !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f && hp->beta2 >= 0.0f && hp->beta2 < 1.0f))
        return fail(BNBQ_EINVAL, "Adam betas must lie in [0, 1)");
    if (opt == BNBQ_RMSPROP && !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f))
        return fail(BNBQ_EINVAL, "RMSprop alpha (beta1) must lie in [0, 1)");

    std::lock_guard<std::mutex> lk(g_na_mu);  // one host staging array for all threads
    StepDesc* descs = g_na_host;
    int nd = 0;
    int64_t blocks = 0;
    bool any8 = false;
    for (int i = 0; i < ntensors; i++) {
        const bnbq_tensor& t = list[i];
        if (t.n < 0) return fail(BNBQ_EINVAL, "tensor %d: n < 0", i);
        if (t.n == 0) continue;
        if (nd == kNoAllocMaxTensors)
            return fail(BNBQ_EINVAL, "bnbq_step_8bit_noalloc takes at most %d non-empty tensors per call "
                        "(its descriptor table is a fixed %d-entry array); split the list or use bnbq_step_8bit",
                        kNoAllocMaxTensors, kNoAllocMaxTensors);
        if (t.state_bits != 8 && t.state_bits != 32) return fail(BNBQ_EINVAL, "tensor %d: state_bits %d not 8 or 32", i, t.state_bits);
        if (t.g_dtype != BNBQ_F32 && t.g_dtype != BNBQ_BF16) return fail(BNBQ_EINVAL, "tensor %d: g_dtype %d unknown", i, t.g_dtype);
        if (!t.p || !t.g || !t.state1 || (two && !t.state2)) return fail(BNBQ_EINVAL, "tensor %d: NULL p, g or state", i);
        if (!aligned_na(t.p, 16)) return fail(BNBQ_EINVAL, "tensor %d: p not 16-byte aligned", i);
        const uintptr_t ga = t.g_dtype == BNBQ_BF16 ? 8 : 16;
        if (!aligned_na(t.g, ga)) return fail(BNBQ_EINVAL, "tensor %d: g not %d-byte aligned", i, (int)ga);
        const uintptr_t sa = t.state_bits == 8 ? 4 : 16;
        if (!aligned_na(t.state1, sa) || (two && !aligned_na(t.state2, sa)))
            return fail(BNBQ_EINVAL, "tensor %d: state not %d-byte aligned", i, (int)sa);
        if (t.state_bits == 8) {
            any8 = true;
            if (!t.absmax1 || (two && !t.absmax2)) return fail(BNBQ_EINVAL, "tensor %d: NULL absmax", i);
            if (!aligned_na(t.absmax1, 4) || (two && !aligned_na(t.absmax2, 4)))
                return fail(BNBQ_EINVAL, "tensor %d: absmax not 4-byte aligned", i);
        }
        StepDesc& d = descs[nd++];
        d.p = t.p;
        d.g = t.g;
        d.s1 = t.state1;
        d.s2 = two ? t.state2 : nullptr;
        d.a1 = t.state_bits == 8 ? t.absmax1 : nullptr;
        d.a2 = (t.state_bits == 8 && two) ? t.absmax2 : nullptr;
        d.n = t.n;
        d.first_block = (int32_t)blocks;
        d.flags = (t.g_dtype == BNBQ_BF16 ? kDescGBf16 : 0) | (t.state_bits == 8 ? kDescState8 : 0);
        blocks += (t.n + blocksize - 1) / blocksize;
        if (blocks > 0x7fff0000LL) return fail(BNBQ_EUNSUPPORTED, "more than 2^31 - 2^16 blocks in one step");
    }
    if (any8) {
        if (!code1 || (two && !code2)) return fail(BNBQ_EINVAL, "8-bit state needs code1%s", two ? " and code2" : "");
        if (!aligned_na(code1, 4) || (two && !aligned_na(code2, 4))) return fail(BNBQ_EINVAL, "codebook not 4-byte aligned");
    }
    if (nd == 0) return BNBQ_OK;
    if (any8) {  // the codebooks must be device memory of this device (checked before any launch)
        bnbq_status cst = check_device_array(code1, 256 * sizeof(float), "code1");
        if (cst == BNBQ_OK && two) cst = check_device_array(code2, 256 * sizeof(float), "code2");
        if (cst != BNBQ_OK) return cst;
    }

    // Scalars formed in double and rounded once to binary32 (same rule as bnbq_step_8bit).
    StepScalars sc;
    const double b1 = hp->beta1, b2 = hp->beta2;
    sc.b1 = hp->beta1;
    sc.b2 = hp->beta2;
    sc.omb1 = (float)(1.0 - b1);
    sc.omb2 = (float)(1.0 - b2);
    sc.step_size = two ? (float)((double)hp->lr / (1.0 - pow(b1, (double)step))) : 0.0f;
    sc.sqrt_bc2 = two ? (float)sqrt(1.0 - pow(b2, (double)step)) : 1.0f;
    volatile float one = 1.0f;
    sc.rcp_sqrt_bc2 = one / sc.sqrt_bc2;
    if (two && !(sc.sqrt_bc2 >= 0x1p-60f && sc.sqrt_bc2 <= 1.0f))
        return fail(BNBQ_EINVAL, "sqrt(1 - beta2^step) = %g outside [2^-60, 1]", (double)sc.sqrt_bc2);
    sc.decay = (opt == BNBQ_ADAMW || opt == BNBQ_LION) ? (float)(1.0 - (double)hp->lr * (double)hp->weight_decay)
                                                       : 1.0f;
    sc.lr = hp->lr;
    sc.eps = hp->eps;
    sc.wd = hp->weight_decay;
    sc.upd_fast = update_fast_allowed(sc.eps, sc.sqrt_bc2) ? 1 : 0;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    bnbq_status st = refuse_capture(s);
    if (st != BNBQ_OK) return st;
    StepDesc* d_table = nullptr;
    st = table_address(&d_table);
    if (st != BNBQ_OK) return st;
    // From pageable host memory: the copy is ordered on `s`, and the host buffer may be reused as
    // soon as the call returns.
    cudaError_t e = cudaMemcpyAsync(d_table, descs, (size_t)nd * sizeof(StepDesc), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_status(e, "descriptor table upload");
    return launch_step(opt, d_table, nd, (int)blocks, sc, any8 ? code1 : nullptr, any8 && two ? code2 : nullptr,
                       blocksize, s);
}
