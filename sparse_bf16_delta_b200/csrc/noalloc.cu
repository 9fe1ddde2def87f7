// noalloc.cu -- dws_encode_noalloc: the fused encode for callers that cannot
// allocate device memory.
//
// Some callers have no way to give libdws a workspace: code that runs inside
// another framework's memory pool, where every device allocation must go
// through an allocator they do not control (or is forbidden outright), and
// latency-critical paths where a cudaMalloc and its implicit device-wide
// synchronisation are not acceptable.  For them, this entry point keeps the
// encode's scratch (the tables of a one-call plan, the scan state and the
// tile descriptors) in a file-scope device array that every GPU loading the
// library holds until the process exits.  The caller passes only inputs and
// outputs.
//
// Limits: at most kNoAllocMaxTensors tensors and kNoAllocMaxTiles tiles of
// 8192 elements (536,870,912 elements in total); larger requests are refused
// with DWS_ERR_WORKSPACE before anything is enqueued.
//
// Every call uses the same array and leaves its contents behind; each call
// rewrites the header and tables and clears the scan state before the
// encode kernel reads them.  Calls that overlap on the GPU (different streams,
// or devices sharing nothing but this file) race on the array of their
// device: order them on one stream or with events.
//
// The first call on a device looks up the array's device address there
// (cudaGetSymbolAddress with that device current); make that first call
// before capturing any stream on that device.  Only a successful lookup is
// kept: after a failed one (say, during a capture) the call returns
// DWS_ERR_CUDA and the next call on that device tries again.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kNoAllocMaxTensors = 256;
constexpr long long kNoAllocMaxTiles = 65536;
constexpr size_t kNoAllocScratchBytes = 5u << 20;  // 5 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu[kMaxDevices];
std::atomic<void *> g_addr[kMaxDevices];  // null until a lookup on that device succeeds

// The scratch array's address on device `dev` (the current device), or null
// if the lookup failed; a failure is not remembered.
void *scratch_address(int dev) {
    void *ptr = g_addr[dev].load(std::memory_order_acquire);
    if (ptr != nullptr) return ptr;
    std::lock_guard<std::mutex> lock(g_addr_mu[dev]);
    ptr = g_addr[dev].load(std::memory_order_relaxed);
    if (ptr != nullptr) return ptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
        (void)cudaGetLastError();  // not left for the next launch check to find
        return nullptr;
    }
    g_addr[dev].store(ptr, std::memory_order_release);
    return ptr;
}

// Tables of a one-call plan, passed by value to the set-up kernel.
struct NoAllocTables {
    long long numel[kNoAllocMaxTensors];
    int num_tensors;
    long long num_tiles;
    unsigned long long fingerprint;
};

// Writes the header (magic, fingerprint, sizes; status, detail and the scan
// counters cleared) and the numel / first_tile tables.
__global__ void noalloc_setup_kernel(WsView ws, NoAllocTables tab) {
    if (threadIdx.x != 0) return;
    WsHeader *h = ws.hdr;
    h->magic = kWsMagic;
    h->fingerprint = tab.fingerprint;
    h->num_tiles = tab.num_tiles;
    h->num_tensors = tab.num_tensors;
    h->status = 0u;
    h->detail = 0;
    h->ticket = 0ull;
    h->abort = 0u;
    h->delta_bad = 0u;
    long long *numel = const_cast<long long *>(ws.numel);
    long long *first = const_cast<long long *>(ws.first_tile);
    long long acc = 0;
    for (int t = 0; t < tab.num_tensors; ++t) {
        numel[t] = tab.numel[t];
        first[t] = acc;
        acc += (tab.numel[t] == 0) ? 1 : (tab.numel[t] + kTileElems - 1) / kTileElems;
    }
    first[tab.num_tensors] = acc;
}

// Copies the call's device status word and detail to the caller's output.
__global__ void noalloc_status_kernel(WsView ws, long long *out) {
    if (threadIdx.x == 0) {
        out[0] = static_cast<long long>(ws.hdr->status);
        out[1] = ws.hdr->detail;
    }
}

}  // namespace
}  // namespace dws

extern "C" DWS_API dws_status_t dws_encode_noalloc(const int64_t *numels, int32_t num_tensors,
                                                   const void *const *old_ptrs,
                                                   const void *const *new_ptrs, int64_t *offsets,
                                                   int32_t *indices, uint16_t *values,
                                                   int64_t capacity, int64_t *status_out,
                                                   dws_stream_t stream) {
    using namespace dws;
    if (numels == nullptr || num_tensors <= 0 || old_ptrs == nullptr || new_ptrs == nullptr ||
        offsets == nullptr || capacity < 0)
        return DWS_ERR_INVALID;
    if (capacity > 0 && (indices == nullptr || values == nullptr)) return DWS_ERR_INVALID;
    if (num_tensors > kNoAllocMaxTensors) return DWS_ERR_WORKSPACE;

    NoAllocTables tab;
    long long tiles = 0;
    unsigned long long h = 0x4e4f414c4c4f4321ull;  // any value both sides agree on
    for (int32_t t = 0; t < num_tensors; ++t) {
        const int64_t n = numels[t];
        if (n < 0 || n > INT32_MAX) return DWS_ERR_INVALID;
        tab.numel[t] = n;
        tiles += (n == 0) ? 1 : (n + kTileElems - 1) / kTileElems;
        h = (h ^ static_cast<unsigned long long>(n)) * 0x100000001b3ull;
    }
    if (tiles > kNoAllocMaxTiles) return DWS_ERR_WORKSPACE;
    const WsLayout L = ws_layout(num_tensors, tiles);
    if (L.total > kNoAllocScratchBytes) return DWS_ERR_WORKSPACE;
    tab.num_tensors = num_tensors;
    tab.num_tiles = tiles;
    tab.fingerprint = h;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DWS_ERR_CUDA;
    void *scratch = scratch_address(dev);
    if (scratch == nullptr) return DWS_ERR_CUDA;

    unsigned char *base = static_cast<unsigned char *>(scratch);
    WsView v;
    v.hdr = reinterpret_cast<WsHeader *>(base);
    v.numel = reinterpret_cast<const long long *>(base + L.numel_off);
    v.first_tile = reinterpret_cast<const long long *>(base + L.first_tile_off);
    v.tile_tensor = reinterpret_cast<const int *>(base + L.tile_tensor_off);
    v.tile_status = reinterpret_cast<unsigned long long *>(base + L.tile_status_off);
    v.tile_desc = reinterpret_cast<TileDesc *>(base + L.tile_desc_off);
    v.num_tiles = tiles;
    v.num_tensors = num_tensors;
    v.fingerprint = h;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    noalloc_setup_kernel<<<1, 32, 0, s>>>(v, tab);
    if (launched() != cudaSuccess) return DWS_ERR_CUDA;
    if (launch_fill_tile_map(v, s) != cudaSuccess) return DWS_ERR_CUDA;
    if (launch_encode(v, reinterpret_cast<const uint16_t *const *>(old_ptrs),
                      reinterpret_cast<const uint16_t *const *>(new_ptrs),
                      reinterpret_cast<long long *>(offsets), reinterpret_cast<int *>(indices),
                      values, capacity, true, 0, -1, s) != cudaSuccess)
        return DWS_ERR_CUDA;
    if (status_out != nullptr) {
        noalloc_status_kernel<<<1, 32, 0, s>>>(v, reinterpret_cast<long long *>(status_out));
        if (launched() != cudaSuccess) return DWS_ERR_CUDA;
    }
    return DWS_OK;
}
