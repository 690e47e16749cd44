// bnbq_api.cu -- the extern "C" entry points of include/bnbq.h: argument checks, host-side
// scalar derivation, the cached descriptor table of the multi-tensor step, codebook
// construction, the device flag word and error reporting.
//
// Sources: "8-bit Optimizers via Block-wise Quantization" (abstract, quoted on the page
// "Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略", section 2) for the method;
// the same page, section "如果需要高精度的参数", for tensors that keep 32-bit state; the page
// "Bitsandbytes" (transformers docs), section "Normal Float 4 (NF4)", for NF4.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "bnbq_internal.h"

// Device flag word (one per device; see bnbq_device_flags).
__device__ unsigned int g_bnbq_flags;

namespace bnbq {

static thread_local std::string t_err;

bnbq_status fail(bnbq_status st, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_err = buf;
    return st;
}

bnbq_status cuda_status(cudaError_t e, const char* what)
{
    if (e == cudaSuccess) return BNBQ_OK;
    return fail(BNBQ_ECUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bnbq_status refuse_capture(cudaStream_t s)
{
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_status(e, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone)
        return fail(BNBQ_EUNSUPPORTED, "the stream is being captured: a step's scalars (bias corrections) and "
                                       "descriptor table belong to one call, so launch it outside the capture");
    return BNBQ_OK;
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
unsigned* g_flag_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

bnbq_status current_device(int* dev)
{
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (*dev < 0 || *dev >= kMaxDevices) return fail(BNBQ_EUNSUPPORTED, "device ordinal %d", *dev);
    return BNBQ_OK;
}
}  // namespace

bnbq_status device_flag_ptr(unsigned** out)
{
    int dev = 0;
    bnbq_status st = current_device(&dev);
    if (st != BNBQ_OK) return st;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_flag_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_bnbq_flags);
        if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(flags)");
        g_flag_ptr[dev] = static_cast<unsigned*>(p);
    }
    *out = g_flag_ptr[dev];
    return BNBQ_OK;
}

bnbq_status sm_count(int* out)
{
    int dev = 0;
    bnbq_status st = current_device(&dev);
    if (st != BNBQ_OK) return st;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_sms[dev]) {
        int v = 0;
        cudaError_t e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_status(e, "cudaDeviceGetAttribute(SM count)");
        g_sms[dev] = v;
    }
    *out = g_sms[dev];
    return BNBQ_OK;
}

namespace {
// cuMemGetAddressRange (driver API, v2 signature), fetched through the runtime so the library
// needs no link against libcuda; null if unavailable.
typedef int (*AddressRangeFn)(unsigned long long* base, size_t* size, unsigned long long ptr);
AddressRangeFn address_range_fn()
{
    static AddressRangeFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<AddressRangeFn>(f);
    }();
    return fn;
}
}  // namespace

bnbq_status check_device_array(const void* p, size_t bytes, const char* name)
{
    int dev = 0;
    bnbq_status st = current_device(&dev);
    if (st != BNBQ_OK) return st;
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();  // a failed query leaves a (non-sticky) error behind; clear it
        return fail(BNBQ_EINVAL, "%s: not a CUDA device pointer (%s)", name, cudaGetErrorString(e));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(BNBQ_EINVAL, "%s: must be device memory of the current device (it is %s memory)", name,
                    attr.type == cudaMemoryTypeHost ? "page-locked host" : "ordinary host");
    if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
        return fail(BNBQ_EINVAL, "%s: lives on device %d but the current device is %d", name, attr.device, dev);
    if (AddressRangeFn range = address_range_fn()) {
        unsigned long long base = 0;
        size_t size = 0;
        if (range(&base, &size, reinterpret_cast<unsigned long long>(p)) == 0) {
            const unsigned long long a = reinterpret_cast<unsigned long long>(p);
            if (a + bytes > base + size)
                return fail(BNBQ_EINVAL, "%s: %zu bytes from this pointer run past the end of its allocation", name, bytes);
        } else {
            cudaGetLastError();
        }
    }
    return BNBQ_OK;
}

// ------------------------------------------------------------------------------------------
// argument checks
// ------------------------------------------------------------------------------------------
namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_blocksize(int B) { return B == 256 || B == 2048 || B == 4096; }
bool valid_q_blocksize(int B) { return B == 64 || B == 128 || valid_blocksize(B); }
bool valid_dtype(int d) { return d == BNBQ_F32 || d == BNBQ_BF16; }
uintptr_t dtype_align(int d) { return d == BNBQ_BF16 ? 8 : 16; }

bnbq_status check_common(const float* code, int K, int64_t n, int B)
{
    if (!code) return fail(BNBQ_EINVAL, "code is NULL");
    if (K != 256 && K != 16) return fail(BNBQ_EINVAL, "code_size %d not in {16, 256}", K);
    if (!aligned(code, 4)) return fail(BNBQ_EINVAL, "code not 4-byte aligned");
    if (n < 0) return fail(BNBQ_EINVAL, "n = %lld < 0", (long long)n);
    if (!valid_q_blocksize(B)) return fail(BNBQ_EINVAL, "blocksize %d not in {64, 128, 256, 2048, 4096}", B);
    return BNBQ_OK;
}

// ------------------------------------------------------------------------------------------
// descriptor-table cache for the multi-tensor step
// ------------------------------------------------------------------------------------------
struct TableEntry {
    int device = -1;
    uint64_t hash = 0;
    std::vector<StepDesc> host;
    StepDesc* d_table = nullptr;
    StepDesc* h_pinned = nullptr;
    cudaEvent_t last_use = nullptr;
    uint64_t tick = 0;
};

constexpr size_t kMaxTables = 8;
std::mutex g_tab_mu;
std::vector<TableEntry> g_tables;
uint64_t g_tick = 0;

uint64_t fnv1a(const void* data, size_t len)
{
    const unsigned char* p = static_cast<const unsigned char*>(data);
    uint64_t h = 1469598103934665603ull;
    for (size_t i = 0; i < len; i++) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}

void free_entry(TableEntry& t)
{
    int cur = -1;
    cudaGetDevice(&cur);
    if (t.device >= 0 && t.device != cur) cudaSetDevice(t.device);
    if (t.last_use) {
        cudaEventSynchronize(t.last_use);
        cudaEventDestroy(t.last_use);
    }
    if (t.d_table) cudaFree(t.d_table);
    if (t.h_pinned) cudaFreeHost(t.h_pinned);
    if (t.device >= 0 && t.device != cur && cur >= 0) cudaSetDevice(cur);
    t = TableEntry();
}

// Find or upload the table for `descs` on the current device; caller holds g_tab_mu.
bnbq_status get_table(const std::vector<StepDesc>& descs, cudaStream_t s, TableEntry** out)
{
    int dev = 0;
    bnbq_status st = current_device(&dev);
    if (st != BNBQ_OK) return st;
    const size_t bytes = descs.size() * sizeof(StepDesc);
    const uint64_t h = fnv1a(descs.data(), bytes);
    for (auto& t : g_tables) {
        if (t.device == dev && t.hash == h && t.host.size() == descs.size() &&
            memcmp(t.host.data(), descs.data(), bytes) == 0) {
            // order this stream after the table's upload (and its last use), which may have been
            // issued on another stream
            cudaError_t e = cudaStreamWaitEvent(s, t.last_use, 0);
            if (e != cudaSuccess) return cuda_status(e, "cudaStreamWaitEvent(descriptor table)");
            t.tick = ++g_tick;
            *out = &t;
            return BNBQ_OK;
        }
    }
    if (g_tables.size() >= kMaxTables) {
        auto lru = std::min_element(g_tables.begin(), g_tables.end(),
                                    [](const TableEntry& a, const TableEntry& b) { return a.tick < b.tick; });
        free_entry(*lru);
        g_tables.erase(lru);
    }
    TableEntry t;
    t.device = dev;
    t.hash = h;
    t.host = descs;
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&t.d_table), bytes);
    if (e != cudaSuccess) return cuda_status(e, "cudaMalloc(descriptor table)");
    e = cudaMallocHost(reinterpret_cast<void**>(&t.h_pinned), bytes);
    if (e != cudaSuccess) {
        cudaFree(t.d_table);
        return cuda_status(e, "cudaMallocHost(descriptor table)");
    }
    memcpy(t.h_pinned, descs.data(), bytes);
    e = cudaEventCreateWithFlags(&t.last_use, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaMemcpyAsync(t.d_table, t.h_pinned, bytes, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaEventRecord(t.last_use, s);
    if (e != cudaSuccess) {
        bnbq_status r = cuda_status(e, "descriptor table upload");
        free_entry(t);
        return r;
    }
    t.tick = ++g_tick;
    g_tables.push_back(std::move(t));
    *out = &g_tables.back();
    return BNBQ_OK;
}

// ------------------------------------------------------------------------------------------
// codebooks (host construction; the CPU test oracle has its own, independent construction)
// ------------------------------------------------------------------------------------------

// binary32 nearest to num/den (0 < num/den <= 1), ties to even, by exact integer arithmetic.
float rational_to_float(uint64_t num, uint64_t den)
{
    // find s with 2^23 <= num*2^s/den < 2^24
    int s = 0;
    unsigned __int128 N = num, D = den;
    while ((N << s) < (D << 23)) s++;
    while ((N << s) >= (D << 24)) s--;
    unsigned __int128 scaled = N << s;
    uint64_t M = (uint64_t)(scaled / D);
    unsigned __int128 rem = scaled % D;
    if (2 * rem > D || (2 * rem == D && (M & 1))) M++;
    if (M == (1ull << 24)) {
        M >>= 1;
        s--;
    }
    return ldexpf((float)M, -s);
}

// Dynamic tree code, decoded pattern by pattern.  A magnitude field of `bits` bits reads: E
// leading zeros, an indicator 1, then f = bits-1-E fraction bits holding k; its value is
// 10^-E * (1/10 + 9/10 * (k+1)/2^f) = (2^f + 9(k+1)) / (2^f * 10^(E+1)).  All zeros is 0.
float dynamic_magnitude(unsigned field, int bits)
{
    if (field == 0) return 0.0f;
    int E = 0;
    while (!(field & (1u << (bits - 1 - E)))) E++;
    const int f = bits - 1 - E;
    const uint64_t k = field & ((1u << f) - 1u);
    uint64_t den = 1ull << f;
    for (int i = 0; i <= E; i++) den *= 10;
    return rational_to_float((1ull << f) + 9 * (k + 1), den);
}

void build_dynamic(bool is_signed, float* out)
{
    for (unsigned pat = 0; pat < 256; pat++) {
        if (is_signed) {
            const bool neg = pat & 0x80u;
            const float m = dynamic_magnitude(pat & 0x7fu, 7);
            // the negative-zero pattern carries the next tree level, +1e-7
            out[pat] = (neg && m == 0.0f) ? rational_to_float(1, 10000000) : (neg ? -m : m);
        } else {
            out[pat] = dynamic_magnitude(pat, 8);
        }
    }
    std::sort(out, out + 256);
}

double std_normal_cdf(double x) { return 0.5 * erfc(-x * M_SQRT1_2); }

// Inverse standard normal CDF by Newton's method on the CDF (p in (0, 1), moderate tails).
double std_normal_quantile(double p)
{
    double x = 0.0;
    for (int it = 0; it < 100; it++) {
        const double pdf = exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
        const double dx = (std_normal_cdf(x) - p) / pdf;
        x -= dx;
        if (fabs(dx) <= 1e-17 * (1.0 + fabs(x))) break;
    }
    return x;
}

// NF4: normal quantiles at evenly spaced probabilities -- 7 below 1/2 starting at delta, zero,
// and 8 above 1/2 ending at 1-delta -- scaled so the extremes are -1 and +1
// (QLoRA, T. Dettmers et al., section 3; delta = (1/30 + 1/32)/2).
void build_nf4(float* out)
{
    const double delta = (1.0 / 30.0 + 1.0 / 32.0) / 2.0;
    const double top = std_normal_quantile(1.0 - delta);
    int c = 0;
    for (int k = 0; k < 7; k++) out[c++] = (float)(std_normal_quantile(delta + (0.5 - delta) * k / 7.0) / top);
    out[c++] = 0.0f;
    for (int k = 1; k <= 8; k++) out[c++] = (float)(std_normal_quantile(0.5 + (0.5 - delta) * k / 8.0) / top);
}

// FP4: the E2M1 4-bit float (page "Quantize 🤗 Transformers models", section "FP4 quantization";
// OCP Microscaling Formats v1.0, section 5.3.3) decoded from its 16 bit patterns -- sign, two
// exponent bits with bias 1, one mantissa bit, subnormals at exponent 0 -- divided by the largest
// magnitude 6 and sorted.  The negative-zero pattern, a duplicate of zero, takes the next finer
// subnormal step 0.25 so that the table is strictly increasing.
void build_fp4(float* out)
{
    double v[16];
    for (int b = 0; b < 16; b++) {
        const int sgn = b >> 3, e = (b >> 1) & 3, m = b & 1;
        const double mag = e == 0 ? 0.5 * m : (1.0 + 0.5 * m) * (double)(1 << (e - 1));
        v[b] = (b == 8) ? 0.25 / 6.0 : (sgn ? -mag : mag) / 6.0;
    }
    for (int i = 1; i < 16; i++)
        for (int j = i; j > 0 && v[j - 1] > v[j]; j--) {
            const double t = v[j];
            v[j] = v[j - 1];
            v[j - 1] = t;
        }
    for (int i = 0; i < 16; i++) out[i] = (float)v[i];
}

void build_linear(float* out)
{
    for (int k = 0; k < 256; k++) out[k] = (float)(-1.0 + 2.0 * k / 255.0);
}

}  // namespace
}  // namespace bnbq

using namespace bnbq;

// ==========================================================================================
// extern "C" entry points
// ==========================================================================================
extern "C" {

const char* bnbq_version(void) { return "0.1.0"; }

const char* bnbq_last_error(void) { return t_err.c_str(); }

int bnbq_code_size(bnbq_code_kind kind)
{
    switch (kind) {
        case BNBQ_CODE_DYNAMIC_SIGNED:
        case BNBQ_CODE_DYNAMIC_UNSIGNED:
        case BNBQ_CODE_LINEAR: return 256;
        case BNBQ_CODE_NF4:
        case BNBQ_CODE_FP4: return 16;
        default: return -1;
    }
}

int bnbq_codebook(bnbq_code_kind kind, float* out)
{
    if (!out) return -1;
    switch (kind) {
        case BNBQ_CODE_DYNAMIC_SIGNED: build_dynamic(true, out); return 256;
        case BNBQ_CODE_DYNAMIC_UNSIGNED: build_dynamic(false, out); return 256;
        case BNBQ_CODE_NF4: build_nf4(out); return 16;
        case BNBQ_CODE_FP4: build_fp4(out); return 16;
        case BNBQ_CODE_LINEAR: build_linear(out); return 256;
        default: return -1;
    }
}

bnbq_status bnbq_check_codebook(const float* host_code, int K)
{
    if (!host_code) return fail(BNBQ_EINVAL, "codebook is NULL");
    if (K != 16 && K != 256) return fail(BNBQ_EINVAL, "codebook size %d not in {16, 256}", K);
    for (int j = 0; j < K; j++) {
        if (!(fabsf(host_code[j]) <= 1.0f)) return fail(BNBQ_EINVAL, "code[%d] = %g not finite in [-1, 1]", j, host_code[j]);
        if (j + 1 < K && !(host_code[j] < host_code[j + 1]))
            return fail(BNBQ_EINVAL, "codebook not strictly increasing at %d", j);
    }
    return BNBQ_OK;
}

bnbq_status bnbq_device_flags(uint32_t* out, int clear)
{
    if (!out) return fail(BNBQ_EINVAL, "out is NULL");
    unsigned* p = nullptr;
    bnbq_status st = device_flag_ptr(&p);
    if (st != BNBQ_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "cudaDeviceSynchronize");
    e = cudaMemcpy(out, p, sizeof(unsigned), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "read device flags");
    if (clear) {
        e = cudaMemset(p, 0, sizeof(unsigned));
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_status(e, "clear device flags");
    }
    return BNBQ_OK;
}

bnbq_status bnbq_quantize_blockwise(const float* code, int code_size, const void* A,
                                    bnbq_dtype a_dtype, int64_t n, int blocksize, float* absmax,
                                    uint8_t* out, bnbq_stream_t stream)
{
    bnbq_status st = check_common(code, code_size, n, blocksize);
    if (st != BNBQ_OK) return st;
    if (!valid_dtype(a_dtype)) return fail(BNBQ_EINVAL, "a_dtype %d unknown", (int)a_dtype);
    if (n == 0) return BNBQ_OK;
    if (!A || !absmax || !out) return fail(BNBQ_EINVAL, "A, absmax and out must be non-NULL");
    if (!aligned(A, dtype_align(a_dtype))) return fail(BNBQ_EINVAL, "A not %d-byte aligned", (int)dtype_align(a_dtype));
    if (!aligned(absmax, 4)) return fail(BNBQ_EINVAL, "absmax not 4-byte aligned");
    if (!aligned(out, code_size == 256 ? 4 : 2)) return fail(BNBQ_EINVAL, "out not %d-byte aligned", code_size == 256 ? 4 : 2);
    st = check_device_array(code, sizeof(float) * (size_t)code_size, "code");
    if (st != BNBQ_OK) return st;
    return launch_quantize(code, code_size, A, a_dtype, n, blocksize, absmax, out,
                           reinterpret_cast<cudaStream_t>(stream));
}

bnbq_status bnbq_dequantize_blockwise(const float* code, int code_size, const uint8_t* q,
                                      const float* absmax, int64_t n, int blocksize, void* out,
                                      bnbq_dtype out_dtype, bnbq_stream_t stream)
{
    bnbq_status st = check_common(code, code_size, n, blocksize);
    if (st != BNBQ_OK) return st;
    if (!valid_dtype(out_dtype)) return fail(BNBQ_EINVAL, "out_dtype %d unknown", (int)out_dtype);
    if (n == 0) return BNBQ_OK;
    if (!q || !absmax || !out) return fail(BNBQ_EINVAL, "q, absmax and out must be non-NULL");
    if (!aligned(q, code_size == 256 ? 4 : 2)) return fail(BNBQ_EINVAL, "q not %d-byte aligned", code_size == 256 ? 4 : 2);
    if (!aligned(absmax, 4)) return fail(BNBQ_EINVAL, "absmax not 4-byte aligned");
    if (!aligned(out, dtype_align(out_dtype))) return fail(BNBQ_EINVAL, "out not %d-byte aligned", (int)dtype_align(out_dtype));
    st = check_device_array(code, sizeof(float) * (size_t)code_size, "code");
    if (st != BNBQ_OK) return st;
    return launch_dequantize(code, code_size, q, absmax, n, blocksize, out, out_dtype,
                             reinterpret_cast<cudaStream_t>(stream));
}

bnbq_status bnbq_step_8bit(bnbq_optim opt, const bnbq_tensor* list, int ntensors,
                           const bnbq_hparams* hp, int step, const float* code1,
                           const float* code2, int blocksize, bnbq_stream_t stream)
{
    if (opt < BNBQ_ADAMW || opt > BNBQ_RMSPROP) return fail(BNBQ_EINVAL, "unknown optimizer %d", (int)opt);
    if (ntensors < 0 || ntensors > (1 << 20)) return fail(BNBQ_EINVAL, "ntensors %d out of [0, 2^20]", ntensors);
    if (ntensors > 0 && !list) return fail(BNBQ_EINVAL, "list is NULL");
    if (!hp) return fail(BNBQ_EINVAL, "hp is NULL");
    if (step < 1) return fail(BNBQ_EINVAL, "step %d < 1", step);
    if (!valid_blocksize(blocksize)) return fail(BNBQ_EINVAL, "blocksize %d not in {256, 2048, 4096}", blocksize);
    const float hv[5] = {hp->lr, hp->beta1, hp->beta2, hp->eps, hp->weight_decay};
    for (float x : hv)
        if (!isfinite(x)) return fail(BNBQ_EINVAL, "hyper-parameters must be finite");
    const bool two = (opt == BNBQ_ADAMW || opt == BNBQ_ADAM);
    if (two && !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f && hp->beta2 >= 0.0f && hp->beta2 < 1.0f))
        return fail(BNBQ_EINVAL, "Adam betas must lie in [0, 1)");
    if (opt == BNBQ_RMSPROP && !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f))
        return fail(BNBQ_EINVAL, "RMSprop alpha (beta1) must lie in [0, 1)");

    std::vector<StepDesc> descs;
    descs.reserve(ntensors);
    int64_t blocks = 0;
    bool any8 = false;
    for (int i = 0; i < ntensors; i++) {
        const bnbq_tensor& t = list[i];
        if (t.n < 0) return fail(BNBQ_EINVAL, "tensor %d: n < 0", i);
        if (t.n == 0) continue;
        if (t.state_bits != 8 && t.state_bits != 32) return fail(BNBQ_EINVAL, "tensor %d: state_bits %d not 8 or 32", i, t.state_bits);
        if (!valid_dtype(t.g_dtype)) return fail(BNBQ_EINVAL, "tensor %d: g_dtype %d unknown", i, t.g_dtype);
        if (!t.p || !t.g || !t.state1 || (two && !t.state2)) return fail(BNBQ_EINVAL, "tensor %d: NULL p, g or state", i);
        if (!aligned(t.p, 16)) return fail(BNBQ_EINVAL, "tensor %d: p not 16-byte aligned", i);
        if (!aligned(t.g, dtype_align(t.g_dtype))) return fail(BNBQ_EINVAL, "tensor %d: g not %d-byte aligned", i, (int)dtype_align(t.g_dtype));
        const uintptr_t sa = t.state_bits == 8 ? 4 : 16;
        if (!aligned(t.state1, sa) || (two && !aligned(t.state2, sa)))
            return fail(BNBQ_EINVAL, "tensor %d: state not %d-byte aligned", i, (int)sa);
        if (t.state_bits == 8) {
            any8 = true;
            if (!t.absmax1 || (two && !t.absmax2)) return fail(BNBQ_EINVAL, "tensor %d: NULL absmax", i);
            if (!aligned(t.absmax1, 4) || (two && !aligned(t.absmax2, 4)))
                return fail(BNBQ_EINVAL, "tensor %d: absmax not 4-byte aligned", i);
        }
        StepDesc d;
        d.p = t.p;
        d.g = t.g;
        d.s1 = t.state1;
        d.s2 = two ? t.state2 : nullptr;
        d.a1 = t.state_bits == 8 ? t.absmax1 : nullptr;
        d.a2 = (t.state_bits == 8 && two) ? t.absmax2 : nullptr;
        d.n = t.n;
        d.first_block = (int32_t)blocks;
        d.flags = (t.g_dtype == BNBQ_BF16 ? kDescGBf16 : 0) | (t.state_bits == 8 ? kDescState8 : 0);
        descs.push_back(d);
        blocks += (t.n + blocksize - 1) / blocksize;
        if (blocks > 0x7fff0000LL) return fail(BNBQ_EUNSUPPORTED, "more than 2^31 - 2^16 blocks in one step");
    }
    if (any8) {
        if (!code1 || (two && !code2)) return fail(BNBQ_EINVAL, "8-bit state needs code1%s", two ? " and code2" : "");
        if (!aligned(code1, 4) || (two && !aligned(code2, 4))) return fail(BNBQ_EINVAL, "codebook not 4-byte aligned");
    }
    if (descs.empty()) return BNBQ_OK;
    if (any8) {  // the codebooks must be device memory of this device (checked before any launch)
        bnbq_status cst = check_device_array(code1, 256 * sizeof(float), "code1");
        if (cst == BNBQ_OK && two) cst = check_device_array(code2, 256 * sizeof(float), "code2");
        if (cst != BNBQ_OK) return cst;
    }

    // Scalars derived once on the host in double and rounded once to binary32.
    StepScalars sc;
    const double b1 = hp->beta1, b2 = hp->beta2;
    sc.b1 = hp->beta1;
    sc.b2 = hp->beta2;
    sc.omb1 = (float)(1.0 - b1);
    sc.omb2 = (float)(1.0 - b2);
    sc.step_size = two ? (float)((double)hp->lr / (1.0 - pow(b1, (double)step))) : 0.0f;
    sc.sqrt_bc2 = two ? (float)sqrt(1.0 - pow(b2, (double)step)) : 1.0f;
    if (two && !(sc.sqrt_bc2 > 0.0f)) return fail(BNBQ_EINVAL, "1 - beta2^step rounds to zero");
    volatile float one = 1.0f;  // keep the reciprocal a binary32 division
    sc.rcp_sqrt_bc2 = one / sc.sqrt_bc2;
    // The kernel divides by sqrt(1-b2^t) with the FMA quotient, exact for divisors in
    // [2^-60, 2^100]; any binary32 beta2 < 1 gives sqrt(1-b2^t) >= 2^-12.
    if (two && !(sc.sqrt_bc2 >= 0x1p-60f && sc.sqrt_bc2 <= 1.0f))
        return fail(BNBQ_EINVAL, "sqrt(1 - beta2^step) = %g outside [2^-60, 1]", (double)sc.sqrt_bc2);
    sc.decay = (opt == BNBQ_ADAMW || opt == BNBQ_LION)
                   ? (float)(1.0 - (double)hp->lr * (double)hp->weight_decay)
                   : 1.0f;
    sc.lr = hp->lr;
    sc.eps = hp->eps;
    sc.wd = hp->weight_decay;
    sc.upd_fast = update_fast_allowed(sc.eps, sc.sqrt_bc2) ? 1 : 0;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    bnbq_status st = refuse_capture(s);
    if (st != BNBQ_OK) return st;
    std::lock_guard<std::mutex> lk(g_tab_mu);
    TableEntry* tab = nullptr;
    st = get_table(descs, s, &tab);
    if (st != BNBQ_OK) return st;
    st = launch_step(opt, tab->d_table, (int)descs.size(), (int)blocks, sc, any8 ? code1 : nullptr,
                     any8 && two ? code2 : nullptr, blocksize, s);
    if (st != BNBQ_OK) return st;
    return cuda_status(cudaEventRecord(tab->last_use, s), "cudaEventRecord(table use)");
}

void bnbq_release(void)
{
    std::lock_guard<std::mutex> lk(g_tab_mu);
    for (auto& t : g_tables) free_entry(t);
    g_tables.clear();
}

}  // extern "C"
