// noalloc.cu -- the expert counting sort with library-owned scratch, for callers
// that cannot allocate device memory.
//
// Some hosts cannot give this library device memory for scratch.  For example, a
// plugin may run inside a framework that owns the whole device-memory budget and
// offers it no allocation hook.  Or a latency-critical loop may not tolerate the
// implicit device synchronisation a cudaMalloc can cause.  lmoe_dispatch_noalloc
// serves them: its scratch (the per-32-token presence bitmap and its per-expert
// prefix) lives in a fixed array that every device which loads this library holds
// until the process exits.  The caller passes only inputs and outputs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/lmoe.h"
#include "moe_kernels.cuh"

static_assert(LMOE_DEVERR_BAD_INDEX == lmoe::DEVERR_BAD_INDEX, "public and device error bits agree");
static_assert(LMOE_DEVERR_REPEATED_INDEX == lmoe::DEVERR_REPEATED_INDEX, "public and device error bits agree");

namespace {

constexpr int kNoallocMaxTokens = 8192;
constexpr int kNoallocMaxExperts = 1024;
constexpr int kNoallocWords = kNoallocMaxTokens / 32;
constexpr size_t kNoallocPlane = static_cast<size_t>(kNoallocWords) * kNoallocMaxExperts;
constexpr int kNoallocHeaderWords = 64;

// bitmap plane, prefix plane, header words: 2 MiB + 256 B on every device.
static __device__ __align__(256) uint32_t g_dispatch_scratch[2 * kNoallocPlane + kNoallocHeaderWords];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchAddr {
    CUcontext ctx = nullptr;  // the context the address belongs to
    uint32_t* addr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

// The calling thread's current driver context (nullptr when none is current yet).
CUcontext current_context() {
    std::call_once(g_ctx_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    });
    CUcontext ctx = nullptr;
    if (g_ctx_current == nullptr || g_ctx_current(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Device address of the scratch array in the current context of the current
// device.  In host code the array's name is only a host-side stand-in, so a
// kernel must be handed this address, never `g_dispatch_scratch` itself.  The
// address is looked up once per device, and again when the thread's current
// context is not the one it was looked up in (a reset device gets a new one;
// a thread that has not used the device yet has none until the lookup, which
// makes the device's primary context current).
uint32_t* scratch_on_current_device(int* status) {
    *status = LMOE_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchAddr& slot = g_scratch[dev];
    if (slot.addr == nullptr || ctx == nullptr || slot.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr) return nullptr;
        const CUcontext now = current_context();
        if (now == nullptr) return nullptr;
        slot.addr = static_cast<uint32_t*>(p);
        slot.ctx = now;
    }
    *status = LMOE_OK;
    return slot.addr;
}

}  // namespace

extern "C" int lmoe_dispatch_noalloc(const int32_t* idx, int32_t T, int32_t top_k, int32_t n_total,
                                     int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                     int32_t* err_word, void* stream) {
    if (T < 0 || T > kNoallocMaxTokens) return LMOE_ERR_TOO_MANY_TOKENS;
    if (top_k < 1 || top_k > 32 || n_total < 1 || n_total > kNoallocMaxExperts || top_k > n_total)
        return LMOE_ERR_UNSUPPORTED_SHAPE;
    if (counts == nullptr || offsets == nullptr) return LMOE_ERR_INVALID_ARG;
    if (T > 0 && (idx == nullptr || perm == nullptr || inv == nullptr)) return LMOE_ERR_INVALID_ARG;
    int status = LMOE_OK;
    uint32_t* base = scratch_on_current_device(&status);
    if (base == nullptr) return status;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* bitmap = base;
    uint32_t* prefix = base + kNoallocPlane;
    int* hdr = reinterpret_cast<int*>(base + 2 * kNoallocPlane);
    // The array keeps the previous call's contents: the header (error word and
    // counters) must start at zero; the bitmap and prefix rows a call reads are
    // all rewritten by that call.
    if (cudaMemsetAsync(hdr, 0, kNoallocHeaderWords * sizeof(int), s) != cudaSuccess) return LMOE_ERR_CUDA;
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * n_total, s) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (n_total + 1), s) != cudaSuccess ||
            (err_word != nullptr && cudaMemsetAsync(err_word, 0, sizeof(int32_t), s) != cudaSuccess))
            return LMOE_ERR_CUDA;
        return LMOE_OK;
    }
    const int nwords = (T + 31) / 32;
    const long slots = static_cast<long>(T) * top_k;
    lmoe::dispatch_bitmap_kernel<<<(nwords + 7) / 8, 256, 8 * n_total * 4, s>>>(idx, T, top_k, n_total, bitmap, hdr);
    lmoe::dispatch_expert_scan_kernel<<<(n_total + 7) / 8, 256, 0, s>>>(bitmap, T, n_total, prefix, counts);
    // no FFN experts here: no tile lists, only offsets
    lmoe::dispatch_offsets_kernel<<<1, 1024, 0, s>>>(counts, n_total, 0, 0, offsets, nullptr, nullptr, nullptr, hdr);
    lmoe::dispatch_scatter_kernel<<<static_cast<unsigned>((slots + 7) / 8), 256, 0, s>>>(
        idx, T, top_k, n_total, 0, bitmap, prefix, offsets, nullptr, 0, 0, nullptr, 0, perm, inv);
    // the caller's copy of this call's error bits (the scratch header is cleared by the next call)
    if (err_word != nullptr &&
        cudaMemcpyAsync(err_word, hdr + lmoe::HDR_ERR, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LMOE_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}
