// Allocation-free variant of the cluster sort.
//
// Some callers cannot allocate device memory at the point where they need
// the sort. Examples:
//  - an engine plugin that may only use memory reserved before execution;
//  - a host loop whose memory budget is fixed when it starts;
//  - code that must not call into the CUDA allocator on its hot path.
// For them, ac_cluster_sort_static runs the same stable counting sort as
// ac_cluster_sort, but its scratch (ranks, tile histograms, cluster sizes,
// per-head descriptors) lives in g_sort_scratch. That is a fixed-size array in
// the library's own device memory. Every GPU that loads the library holds it
// until the process exits. The caller passes only the inputs and outputs.
#include <cuda.h>
#include <mutex>

#include "adacluster.h"
#include "ac_kernels.cuh"
#include "ac_multistage.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_sort_scratch[kStaticScratchBytes];

// Device address of g_sort_scratch per device.  In host code the symbol is
// only a host-side stand-in, so the address is looked up per device (with
// that device current) and the kernels get the looked-up pointer.  The
// address belongs to the device's current context: it is looked up again
// when the context's id changes (after cudaDeviceReset, for example).
void *g_scratch_addr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (CtxGetCurrentFn)f;
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (CtxGetIdFn)f;
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

using namespace ac;

extern "C" AC_API ac_status ac_cluster_sort_static(const int32_t *assign, int heads, int n, int cap,
                                                   const int32_t *ncl, int32_t *perm, int32_t *offsets,
                                                   void *stream) {
    if (!assign || !perm || !offsets || heads < 1 || n < 1 || cap < 1) return AC_ERR_INVALID_ARG;
    if (cap > 8192 || (long long)heads * n > 0x3fffffffLL) return AC_ERR_UNSUPPORTED;
    const size_t status_b = 256;
    const size_t seg_b = up256((size_t)heads * sizeof(HeadSeg));
    const size_t rank_b = up256((size_t)heads * n * sizeof(int32_t));
    const size_t cnt_b = up256((size_t)heads * cap * sizeof(int32_t));
    const size_t hist_b = up256(sort_hist_elems(heads, n, cap) * sizeof(int32_t));
    if (status_b + seg_b + rank_b + cnt_b + hist_b > kStaticScratchBytes) return AC_ERR_UNSUPPORTED;

    // A launch error left by earlier, unrelated work on this thread would be
    // read back below as this call's; clear it first.
    (void)cudaGetLastError();
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AC_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return AC_ERR_UNSUPPORTED;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        const unsigned long long ctx = current_ctx_id();
        if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_sort_scratch) != cudaSuccess || !p) return AC_ERR_CUDA;
            g_scratch_addr[dev] = p;
            g_scratch_ctx[dev] = ctx;
        }
        base = g_scratch_addr[dev];
    }
    char *b = static_cast<char *>(base);
    int *status = reinterpret_cast<int *>(b);
    HeadSeg *seg = reinterpret_cast<HeadSeg *>(b + status_b);
    int32_t *rank = reinterpret_cast<int32_t *>(b + status_b + seg_b);
    int32_t *cnt = reinterpret_cast<int32_t *>(b + status_b + seg_b + rank_b);
    int32_t *hist = reinterpret_cast<int32_t *>(b + status_b + seg_b + rank_b + cnt_b);

    // Every scratch region below is written by this call before it is read
    // (descriptors, ranks, the histograms of the tiles in use, cluster sizes),
    // so no region has to start at zero.  The status word receives
    // out-of-range ids and clamped counts; it is cleared here so that it
    // describes this call only, and it is not read back.
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(status, 0, status_b, st) != cudaSuccess) return AC_ERR_CUDA;
    k_seg_from_counts(heads, n, ncl, cap, cap, seg, status, st);
    k_sort(assign, nullptr, seg, heads, n, n, cap, rank, hist, cnt, offsets, perm, status, st);
    return cudaGetLastError() == cudaSuccess ? AC_OK : AC_ERR_CUDA;
}
