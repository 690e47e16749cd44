// Exhaustive check of the library's nearest-code search (build_bucket_entries and
// nearest_code_word in bnbq_device.cuh) for one codebook: every binary32 x with |x| <= 1, both
// signs (2,130,706,434 values), against a plain count of the binary32 midpoints below x,
//      q = #{ j : x > mid_j },  mid_j = fl32((code_j + code_{j+1}) / 2)  (sum formed in double),
// with the midpoints formed on the host.  Each search mode is checked where it applies: the
// one-load rule when no bucket holds two midpoints, the non-negative rule when every code is
// >= 0, the midpoint walk always.
//
// Usage: search_exhaustive <codebook file: K raw float32 values> <K>
// Prints one line per mode and a final status line; exits 0 only if every checked mode matches.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../block_wise_bit_b200/csrc/bnbq_device.cuh"

namespace {

constexpr uint32_t kHalfValues = 0x3F800000u + 1u;  // bit patterns 0 .. 0x3F800000 (+0 .. 1.0)

__global__ void setup(const float* code, int K, float* mid, uint32_t* table, int* flags)
{
    bool bad = false, tiny = false;
    bnbq::stage_midpoints(code, mid, K, bad, tiny);
    __syncthreads();
    const bool general = bnbq::build_bucket_entries(table + bnbq::kHalf, mid, K, -bnbq::kHalf, bnbq::kHalf - 1);
    const int g = __syncthreads_or(general);
    const int b = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        flags[0] = g;
        flags[1] = b;
    }
}

template <int MODE>
__global__ void sweep(const uint32_t* table, const float* mid, const float* ref_mid, int K,
                      unsigned long long* bad, unsigned* first)
{
    __shared__ float rm[256];
    for (int j = threadIdx.x; j < K - 1; j += blockDim.x) rm[j] = ref_mid[j];
    __syncthreads();
    const uint32_t* center = table + bnbq::kHalf;
    const uint64_t total = 2ull * kHalfValues;
    unsigned long long n = 0;
    for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < total; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t bits = i < kHalfValues ? (uint32_t)i : 0x80000000u + (uint32_t)(i - kHalfValues);
        const float x = __uint_as_float(bits);
        const uint32_t q = bnbq::nearest_code_word<MODE>(center, mid, x) >> 24;
        uint32_t r = 0;
        for (int j = 0; j < K - 1; j++) r += (x > rm[j]) ? 1u : 0u;
        if (q != r) {
            n++;
            atomicCAS(first, 0xffffffffu, bits);
        }
    }
    if (n) atomicAdd(bad, n);
}

template <int MODE>
bool run_mode(const char* name, const uint32_t* table, const float* mid, const float* ref_mid, int K,
              unsigned long long* d_bad, unsigned* d_first)
{
    cudaMemset(d_bad, 0, sizeof(*d_bad));
    cudaMemset(d_first, 0xff, sizeof(*d_first));
    sweep<MODE><<<148 * 8, 256>>>(table, mid, ref_mid, K, d_bad, d_first);
    const cudaError_t e = cudaDeviceSynchronize();
    unsigned long long bad = ~0ull;
    unsigned first = 0;
    cudaMemcpy(&bad, d_bad, sizeof(bad), cudaMemcpyDeviceToHost);
    cudaMemcpy(&first, d_first, sizeof(first), cudaMemcpyDeviceToHost);
    printf("mode %s status %s mismatches %llu first %08x\n", name, cudaGetErrorString(e), bad, first);
    return e == cudaSuccess && bad == 0;
}

}  // namespace

int main(int argc, char** argv)
{
    if (argc != 3) {
        fprintf(stderr, "usage: %s <codebook.f32> <K>\n", argv[0]);
        return 2;
    }
    const int K = atoi(argv[2]);
    if (K != 16 && K != 256) return 2;
    std::vector<float> code(K);
    FILE* f = fopen(argv[1], "rb");
    if (!f || fread(code.data(), sizeof(float), (size_t)K, f) != (size_t)K) return 2;
    fclose(f);
    std::vector<float> ref_mid(K - 1);
    bool nonneg = true;
    for (int j = 0; j < K; j++) {
        if (code[j] < 0.0f) nonneg = false;
        if (j + 1 < K) ref_mid[j] = (float)(((double)code[j] + (double)code[j + 1]) * 0.5);
    }

    float *d_code = nullptr, *d_mid = nullptr, *d_ref = nullptr;
    uint32_t* d_table = nullptr;
    int* d_flags = nullptr;
    unsigned long long* d_bad = nullptr;
    unsigned* d_first = nullptr;
    if (cudaMalloc(&d_code, 256 * sizeof(float)) != cudaSuccess || cudaMalloc(&d_mid, 256 * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&d_ref, 256 * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&d_table, bnbq::kTableSize * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&d_flags, 2 * sizeof(int)) != cudaSuccess || cudaMalloc(&d_bad, sizeof(*d_bad)) != cudaSuccess ||
        cudaMalloc(&d_first, sizeof(*d_first)) != cudaSuccess)
        return 3;
    cudaMemcpy(d_code, code.data(), K * sizeof(float), cudaMemcpyHostToDevice);
    cudaMemcpy(d_ref, ref_mid.data(), (K - 1) * sizeof(float), cudaMemcpyHostToDevice);
    setup<<<1, 1024>>>(d_code, K, d_mid, d_table, d_flags);
    cudaError_t e = cudaDeviceSynchronize();
    int flags[2] = {-1, -1};
    std::vector<float> dev_mid(K);
    cudaMemcpy(flags, d_flags, sizeof(flags), cudaMemcpyDeviceToHost);
    cudaMemcpy(dev_mid.data(), d_mid, K * sizeof(float), cudaMemcpyDeviceToHost);
    bool mids_equal = true;
    for (int j = 0; j + 1 < K; j++) mids_equal = mids_equal && dev_mid[j] == ref_mid[j];
    printf("setup status %s general %d bad %d nonneg %d midpoints %s\n", cudaGetErrorString(e), flags[0], flags[1],
           nonneg ? 1 : 0, mids_equal ? "equal" : "DIFFER");
    bool ok = e == cudaSuccess && flags[1] == 0 && mids_equal;
    if (ok && flags[0] == 0) ok = run_mode<bnbq::kSearchSigned>("signed", d_table, d_mid, d_ref, K, d_bad, d_first) && ok;
    if (ok && nonneg) ok = run_mode<bnbq::kSearchNonNeg>("nonneg", d_table, d_mid, d_ref, K, d_bad, d_first) && ok;
    if (ok) ok = run_mode<bnbq::kSearchGeneral>("general", d_table, d_mid, d_ref, K, d_bad, d_first) && ok;
    printf("result %s\n", ok ? "ok" : "FAIL");
    return ok ? 0 : 1;
}
