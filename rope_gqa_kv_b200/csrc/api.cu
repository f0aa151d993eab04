// api.cu -- status strings, version, and the bounded-wait self-test of the libgqa C ABI.
#include "common.cuh"
#include "ptx.cuh"

extern "C" const char *gqa_status_string(gqa_status s) {
    switch (s) {
        case GQA_OK: return "ok";
        case GQA_ERR_INVALID_ARG: return "invalid argument (null, size, alignment or Hq % Hkv)";
        case GQA_ERR_UNSUPPORTED: return "unsupported (head_dim must be 64, 96 or 128; sm_100 GPU)";
        case GQA_ERR_CAPACITY: return "positions or lengths exceed the cache capacity Lmax";
        case GQA_ERR_TIMEOUT: return "a bounded wait timed out";
        case GQA_ERR_CUDA: return "CUDA runtime or driver error";
        case GQA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

extern "C" int gqa_version(void) { return 200; }

// One thread waits on an mbarrier that nothing arrives on, through
// ptx::mbar_wait -- the function every kernel of the library waits with -- with
// its limit shortened to limit_ns: the wait gives up, and the thread raises
// GQA_DEV_TIMEOUT instead of hanging.  A second wait, on a barrier whose phase
// has completed, must succeed at once (the success path of the same function).
__global__ void selftest_wait_kernel(int32_t *status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar[2];
    const uint32_t never = gqa::ptx::smem_addr(&bar[0]);
    const uint32_t done = gqa::ptx::smem_addr(&bar[1]);
    gqa::ptx::mbar_init(never, 1);
    gqa::ptx::mbar_init(done, 1);
    gqa::ptx::fence_barrier_init();
    gqa::ptx::mbar_arrive(done);                       // completes phase 0 of `done`
    if (!gqa::ptx::mbar_wait(done, 0, limit_ns)) gqa::report(status, GQA_DEV_BAD_LEN);
    if (!gqa::ptx::mbar_wait(never, 0, limit_ns)) gqa::report(status, GQA_DEV_TIMEOUT);
}

extern "C" gqa_status gqa_selftest_bounded_wait(int32_t *status_dev, int limit_ms, void *stream) {
    if (!status_dev || limit_ms < 1 || limit_ms > 10000) return GQA_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
        status_dev, (unsigned long long)limit_ms * 1000000ull);
    return gqa_host::launch_status();
}
