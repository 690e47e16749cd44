// Check of the library's bulk-copy helpers (bnbq_async.cuh): a 32 KB cp.async.bulk copy into
// shared memory completes its mbarrier and delivers the bytes, and a wait on a barrier phase that
// never completes (a barrier that nothing arrives on) returns false after the wait budget instead
// of spinning on, leaving the context usable for the next launch.
//
// Usage: bulk_copy_wait
// Prints one line per case and a final status line; exits 0 only if every case behaves.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "../../block_wise_bit_b200/csrc/bnbq_async.cuh"

namespace {

constexpr uint32_t kBytes = 32768;

// One CTA: thread 0 copies src[0, kBytes) into shared memory; every thread waits for the phase and
// copies the stage back out; landed[t] = the wait's result.
__global__ void copy_lands(const unsigned char* src, unsigned char* dst, int* landed)
{
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBytes);
    if (threadIdx.x == 0) {
        bnbq::mbar_init(bar, 1);
        bnbq::mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bnbq::mbar_arrive_expect(bar, kBytes);
        bnbq::bulk_copy_g2s(smem, src, kBytes, bar);
    }
    const bool ok = bnbq::mbar_wait(bar, 0);
    landed[threadIdx.x] = ok ? 1 : 0;
    if (ok)
        for (uint32_t i = threadIdx.x; i < kBytes; i += blockDim.x) dst[i] = smem[i];
}

// One CTA: a barrier expecting one arrival that never comes; every thread's bounded wait must give
// up.  gave_up[t] = 1 if the wait returned false.
__global__ void wait_runs_out(int* gave_up)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        bnbq::mbar_init(&bar, 1);
        bnbq::mbar_init_fence();
    }
    __syncthreads();
    gave_up[threadIdx.x] = bnbq::mbar_wait(&bar, 0) ? 0 : 1;
}

bool check(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) printf("%s: %s\n", what, cudaGetErrorString(e));
    return e == cudaSuccess;
}

}  // namespace

int main()
{
    bool ok = true;
    const int threads = 128;
    std::vector<unsigned char> h(kBytes);
    for (uint32_t i = 0; i < kBytes; i++) h[i] = (unsigned char)(i * 131u + 7u);
    unsigned char *src = nullptr, *dst = nullptr;
    int* flags = nullptr;
    if (!check(cudaMalloc(&src, kBytes), "cudaMalloc") || !check(cudaMalloc(&dst, kBytes), "cudaMalloc") ||
        !check(cudaMalloc(&flags, threads * sizeof(int)), "cudaMalloc"))
        return 1;
    ok &= check(cudaMemcpy(src, h.data(), kBytes, cudaMemcpyHostToDevice), "upload");
    ok &= check(cudaMemset(dst, 0, kBytes), "memset");
    const int smem = kBytes + 16;
    ok &= check(cudaFuncSetAttribute(copy_lands, cudaFuncAttributeMaxDynamicSharedMemorySize, smem), "smem attribute");
    copy_lands<<<1, threads, smem>>>(src, dst, flags);
    ok &= check(cudaDeviceSynchronize(), "copy_lands");
    std::vector<unsigned char> back(kBytes);
    std::vector<int> f(threads);
    ok &= check(cudaMemcpy(back.data(), dst, kBytes, cudaMemcpyDeviceToHost), "download");
    ok &= check(cudaMemcpy(f.data(), flags, threads * sizeof(int), cudaMemcpyDeviceToHost), "download");
    int landed = 0;
    for (int v : f) landed += v;
    const bool same = back == h;
    printf("copy landed %d of %d waits, bytes %s\n", landed, threads, same ? "equal" : "differ");
    ok &= landed == threads && same;

    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    cudaEventRecord(e0);
    wait_runs_out<<<1, 32>>>(flags);
    cudaEventRecord(e1);
    ok &= check(cudaDeviceSynchronize(), "wait_runs_out");
    float ms = 0.0f;
    cudaEventElapsedTime(&ms, e0, e1);
    ok &= check(cudaMemcpy(f.data(), flags, 32 * sizeof(int), cudaMemcpyDeviceToHost), "download");
    int gave_up = 0;
    for (int i = 0; i < 32; i++) gave_up += f[i];
    printf("wait gave up %d of 32 after %.0f ms\n", gave_up, ms);
    ok &= gave_up == 32 && ms > 100.0f && ms < 20000.0f;

    // the context is still usable: the copy runs again
    cudaMemset(dst, 0, kBytes);
    copy_lands<<<1, threads, smem>>>(src, dst, flags);
    ok &= check(cudaDeviceSynchronize(), "copy_lands again");
    ok &= check(cudaMemcpy(back.data(), dst, kBytes, cudaMemcpyDeviceToHost), "download");
    printf("copy after the timeout: bytes %s\n", back == h ? "equal" : "differ");
    ok &= back == h;
    cudaFree(src);
    cudaFree(dst);
    cudaFree(flags);
    printf("result %s\n", ok ? "ok" : "FAILED");
    return ok ? 0 : 1;
}
