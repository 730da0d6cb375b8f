// symnmf_sh_noalloc: the S-stream product Y = S X without a caller workspace.
//
// Every other entry point that needs device scratch takes it from the caller
// as a workspace.  Some callers cannot allocate device memory when they call
// in: a host runtime whose device memory is owned entirely by its own pool
// or by another framework's caching allocator (a cudaMalloc from outside
// would fragment it or break its budget), or a latency-critical loop that
// cannot take cudaMalloc's implicit device-wide synchronisation.  For them
// this variant keeps its scratch in a fixed file-scope device array instead.
#include "common.cuh"

namespace symnmf {

// 4 MiB of device scratch.  Every GPU that loads the library holds it until
// the process exits.  It holds the TF32 split of X and the error word.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;
constexpr size_t kNoAllocErrFloats = 64;  // error word slot, kept 256-byte aligned
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Host code cannot use g_noalloc_scratch's name as a device address: it is a
// host-side stand-in.  The device address belongs to the context the module
// was loaded into, so it is looked up on every call, with the calling device
// current: after cudaDeviceReset, or under another context on the same
// device, a cached address would point at memory that is no longer the
// array.  The lookup is a host-side table read once the module is loaded,
// negligible next to a pass over S.
static int noalloc_scratch(float** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
        set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return SYMNMF_ERR_CUDA;
    }
    *out = static_cast<float*>(p);
    return SYMNMF_OK;
}

size_t noalloc_floats_needed(int64_t n, int k) {
    return (size_t)xt_rows(k) * (size_t)xt_ld(n) + kNoAllocErrFloats;
}

}  // namespace symnmf

using namespace symnmf;

extern "C" int symnmf_sh_noalloc(const float* S, int64_t n, int64_t lds, const float* X, int k,
                                 float* Y, symnmf_stream_t stream) {
    clear_error();
    if (n < 1 || lds < n || lds % 4 != 0) {
        set_error("n = %lld, lds = %lld: need n >= 1, lds >= n, lds a multiple of 4", (long long)n,
                  (long long)lds);
        return SYMNMF_ERR_INVALID_ARG;
    }
    // n alone bounds the scratch (one split row per instrument): reject any n
    // the array cannot hold before the size product below is formed, so that
    // product cannot wrap
    if (n > (int64_t)kNoAllocScratchFloats) {
        set_error("symnmf_sh_noalloc: n = %lld exceeds the static scratch of %zu floats; "
                  "use symnmf_sh with a workspace",
                  (long long)n, kNoAllocScratchFloats);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (lds > (int64_t(1) << 62) / n) {
        set_error("n * lds overflows");
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (S == nullptr || (reinterpret_cast<uintptr_t>(S) & 15u) != 0) {
        set_error("S must be a non-null 16-byte aligned device pointer");
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (k < 1 || k > KMAX) {
        set_error("k = %d must be in [1, %d]", k, KMAX);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (X == nullptr || Y == nullptr || (reinterpret_cast<uintptr_t>(X) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(Y) & 3u) != 0) {
        set_error("X and Y must be non-null 4-byte aligned device pointers");
        return SYMNMF_ERR_INVALID_ARG;
    }
    const size_t need = noalloc_floats_needed(n, k);
    if (need > kNoAllocScratchFloats) {
        set_error("symnmf_sh_noalloc: n = %lld with k = %d needs %zu floats of static scratch; "
                  "the limit is %zu (2 * roundup(k, 8) * roundup(n, 32) + 64 <= 1048576); "
                  "use symnmf_sh with a workspace",
                  (long long)n, k, need, kNoAllocScratchFloats);
        return SYMNMF_ERR_INVALID_ARG;
    }
    Dev d;
    SYMNMF_TRY(device_info(&d));
    float* scratch = nullptr;
    SYMNMF_TRY(noalloc_scratch(&scratch));
    cudaStream_t s = (cudaStream_t)stream;
    // one contraction split writes Y directly; no partials
    TcPlan p = plan_stream_tc(d, n, k, 0, n);
    p.splits = 1;
    p.jspan = (p.j1 - p.j0 + 31) / 32 * 32;
    float* XT = scratch + kNoAllocErrFloats;
    int* err = reinterpret_cast<int*>(scratch);
    const int64_t ldxt = xt_ld(n);
    // the array keeps the previous call's contents: the error word starts at zero
    SYMNMF_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), s));
    SYMNMF_TRY(launch_split(X, nullptr, k, k, 0, n, p.j0, p.j1, XT, ldxt, s));
    SYMNMF_TRY(launch_stream_tc(p, S, lds, XT, ldxt, Y, err, nullptr, s));
    // a bounded device-side wait that gave up is reported in the error word
    int h = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (h != 0) {
        set_error("an S-stream pipeline wait timed out on the device (code %d)", h);
        return SYMNMF_ERR_TIMEOUT;
    }
    return SYMNMF_OK;
}
