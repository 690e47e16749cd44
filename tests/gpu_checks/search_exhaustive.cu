// Exhaustive check of the library's nearest-code search (build_bucket_entries and
// nearest_code_word in bnbq_device.cuh) for one codebook: every binary32 x with |x| <= 1, both
// signs (2,130,706,434 values), against a plain count of the binary32 midpoints below x,
//      q = #{ j : x > mid_j },  mid_j = fl32((code_j + code_{j+1}) / 2)  (sum formed in double),
// with the midpoints formed on the host.  Each search mode is checked where it applies: the
// one-load rule when no bucket holds two midpoints, the non-negative rule when every code is
// >= 0, the midpoint walk always, for a 16-entry codebook the 11-bit-prefix table
// (build_table11 / nearest_code_word11) when none of its buckets holds two midpoints, and the
// one-load rule with the sign on the FMA pipe (bnbq_search_fma.cuh: the table's negative half
// biased, nearest_code_word_fma) wherever the one-load rule applies.
//
// Usage: search_exhaustive <codebook file: K raw float32 values> <K>
// Prints one line per mode and a final status line; exits 0 only if every checked mode matches.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../block_wise_bit_b200/csrc/bnbq_device.cuh"
#include "../../block_wise_bit_b200/csrc/bnbq_search_fma.cuh"

namespace {

constexpr uint32_t kHalfValues = 0x3F800000u + 1u;  // bit patterns 0 .. 0x3F800000 (+0 .. 1.0)

__global__ void setup(const float* code, int K, float* mid, uint32_t* table, uint32_t* table11, int* flags)
{
    bool bad = false, tiny = false;
    bnbq::stage_midpoints(code, mid, K, bad, tiny);
    __syncthreads();
    const bool general = bnbq::build_bucket_entries(table + bnbq::kHalf, mid, K, -bnbq::kHalf, bnbq::kHalf - 1);
    const bool general11 = K == 16 && bnbq::build_table11(table11, mid, K);
    const int g = __syncthreads_or(general);
    const int g11 = __syncthreads_or(general11);
    const int b = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        flags[0] = g;
        flags[1] = b;
        flags[2] = g11;
    }
}

// One pass over every value: the reference count is formed once per value and compared with each
// search mode that applies (check[m] != 0), mismatches counted per mode.
constexpr int kModes = 5;
struct Checks {
    int on[kModes];
};

// A copy of the table with the negative half biased, for the FMA-pipe search.
__global__ void bias_copy(const uint32_t* table, uint32_t* biased)
{
    for (int i = threadIdx.x; i < bnbq::kTableSize; i += blockDim.x) biased[i] = table[i];
    __syncthreads();
    bnbq::bias_negative_half(biased);
}

__global__ void sweep(const uint32_t* table, const uint32_t* table11, const uint32_t* biased, const float* mid,
                      const float* ref_mid, int K, Checks check, unsigned long long* bad, unsigned* first)
{
    __shared__ float rm[256];
    for (int j = threadIdx.x; j < K - 1; j += blockDim.x) rm[j] = ref_mid[j];
    __syncthreads();
    const uint32_t* center = table + bnbq::kHalf;
    const uint32_t* center_b = biased + bnbq::kHalf;
    const uint64_t total = 2ull * kHalfValues;
    unsigned long long n[kModes] = {0, 0, 0, 0, 0};
    for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < total; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t bits = i < kHalfValues ? (uint32_t)i : 0x80000000u + (uint32_t)(i - kHalfValues);
        const float x = __uint_as_float(bits);
        uint32_t r = 0;
        for (int j = 0; j < K - 1; j++) r += (x > rm[j]) ? 1u : 0u;
        uint32_t q[kModes] = {r, r, r, r, r};
        if (check.on[0]) q[0] = bnbq::nearest_code_word<bnbq::kSearchSigned>(center, mid, x) >> 24;
        if (check.on[1]) q[1] = bnbq::nearest_code_word<bnbq::kSearchNonNeg>(center, mid, x) >> 24;
        if (check.on[2]) q[2] = bnbq::nearest_code_word<bnbq::kSearchGeneral>(center, mid, x) >> 24;
        if (check.on[3]) q[3] = bnbq::nearest_code_word11(table11, x) >> 24;
        if (check.on[4]) q[4] = bnbq::nearest_code_word_fma(center_b, x) >> 24;
#pragma unroll
        for (int m = 0; m < kModes; m++)
            if (q[m] != r) {
                n[m]++;
                atomicCAS(&first[m], 0xffffffffu, bits);
            }
    }
    for (int m = 0; m < kModes; m++)
        if (n[m]) atomicAdd(&bad[m], n[m]);
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
    uint32_t *d_table = nullptr, *d_table11 = nullptr, *d_biased = nullptr;
    int* d_flags = nullptr;
    unsigned long long* d_bad = nullptr;
    unsigned* d_first = nullptr;
    if (cudaMalloc(&d_code, 256 * sizeof(float)) != cudaSuccess || cudaMalloc(&d_mid, 256 * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&d_ref, 256 * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&d_table, bnbq::kTableSize * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&d_table11, bnbq::kTable11 * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&d_biased, bnbq::kTableSize * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&d_flags, 3 * sizeof(int)) != cudaSuccess || cudaMalloc(&d_bad, 5 * sizeof(*d_bad)) != cudaSuccess ||
        cudaMalloc(&d_first, 5 * sizeof(*d_first)) != cudaSuccess)
        return 3;
    cudaMemcpy(d_code, code.data(), K * sizeof(float), cudaMemcpyHostToDevice);
    cudaMemcpy(d_ref, ref_mid.data(), (K - 1) * sizeof(float), cudaMemcpyHostToDevice);
    setup<<<1, 1024>>>(d_code, K, d_mid, d_table, d_table11, d_flags);
    cudaError_t e = cudaDeviceSynchronize();
    int flags[3] = {-1, -1, -1};
    std::vector<float> dev_mid(K);
    cudaMemcpy(flags, d_flags, sizeof(flags), cudaMemcpyDeviceToHost);
    cudaMemcpy(dev_mid.data(), d_mid, K * sizeof(float), cudaMemcpyDeviceToHost);
    bool mids_equal = true;
    for (int j = 0; j + 1 < K; j++) mids_equal = mids_equal && dev_mid[j] == ref_mid[j];
    printf("setup status %s general %d bad %d nonneg %d prefix11-general %d midpoints %s\n", cudaGetErrorString(e),
           flags[0], flags[1], nonneg ? 1 : 0, flags[2], mids_equal ? "equal" : "DIFFER");
    bool ok = e == cudaSuccess && flags[1] == 0 && mids_equal;
    if (ok) {
        // the one-load rule where no bucket holds two midpoints (and its FMA-pipe form), the
        // non-negative rule for a codebook without negative codes, the midpoint walk always, and
        // for 16 codes the 11-bit-prefix table where none of its buckets holds two midpoints
        Checks check = {{flags[0] == 0 ? 1 : 0, nonneg ? 1 : 0, 1, (K == 16 && flags[2] == 0) ? 1 : 0,
                         flags[0] == 0 ? 1 : 0}};
        bias_copy<<<1, 1024>>>(d_table, d_biased);
        cudaMemset(d_bad, 0, 5 * sizeof(*d_bad));
        cudaMemset(d_first, 0xff, 5 * sizeof(*d_first));
        sweep<<<148 * 8, 256>>>(d_table, d_table11, d_biased, d_mid, d_ref, K, check, d_bad, d_first);
        e = cudaDeviceSynchronize();
        unsigned long long bad[kModes] = {~0ull, ~0ull, ~0ull, ~0ull, ~0ull};
        unsigned first[kModes] = {0, 0, 0, 0, 0};
        cudaMemcpy(bad, d_bad, sizeof(bad), cudaMemcpyDeviceToHost);
        cudaMemcpy(first, d_first, sizeof(first), cudaMemcpyDeviceToHost);
        const char* names[kModes] = {"signed", "nonneg", "general", "prefix11", "signed-fma"};
        for (int m = 0; m < kModes; m++)
            if (check.on[m]) {
                printf("mode %s status %s mismatches %llu first %08x\n", names[m], cudaGetErrorString(e), bad[m],
                       first[m]);
                ok = ok && e == cudaSuccess && bad[m] == 0;
            }
    }
    printf("result %s\n", ok ? "ok" : "FAIL");
    return ok ? 0 : 1;
}
