// dws_abi.cu -- the libdws C ABI (declared in include/dws.h): host-side
// validation, the plan (multi-tensor descriptor table), workspace upload,
// kernel launches, the two-stream XOR layer pipeline and status readback.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "dws_internal.cuh"

namespace dws {
size_t encode_smem_bytes();
cudaError_t encode_set_attributes();
cudaError_t encode_occupancy(int *ctas_per_sm);

namespace {
constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
DeviceInfo g_info[kMaxDevices];
cudaError_t g_err[kMaxDevices];

void init_device(int dev) {
    DeviceInfo di{};
    cudaError_t e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    int l2 = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    di.l2_bytes = l2;
    if (e == cudaSuccess) e = encode_set_attributes();
    if (e == cudaSuccess) e = encode_occupancy(&di.encode_ctas_per_sm);
    if (e == cudaSuccess) {
        if (di.encode_ctas_per_sm < 1) di.encode_ctas_per_sm = 1;
    }
    g_info[dev] = di;
    g_err[dev] = e;
}
}  // namespace

namespace {
std::atomic<unsigned long long> g_launches{0};
}

cudaError_t launched() {
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

cudaError_t device_info(DeviceInfo *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_once[dev], init_device, dev);
    if (g_err[dev] != cudaSuccess) return g_err[dev];
    *out = g_info[dev];
    return cudaSuccess;
}

}  // namespace dws

using dws::WsHeader;
using dws::WsLayout;
using dws::WsView;

struct dws_plan {
    int32_t T;
    int64_t N;
    int64_t ntiles;
    uint64_t fingerprint;
    WsLayout layout;
    std::vector<unsigned char> image;  // header + numel + first_tile, as uploaded
};

bool dws::plan_numels(const dws_plan_t *plan, int32_t *num_tensors, const long long **numels) {
    if (plan == nullptr) return false;
    *num_tensors = plan->T;
    *numels = reinterpret_cast<const long long *>(plan->image.data() + plan->layout.numel_off);
    return true;
}

namespace {

uint64_t fnv1a(uint64_t h, uint64_t v) {
    for (int i = 0; i < 8; ++i) {
        h ^= (v >> (8 * i)) & 0xffu;
        h *= 0x100000001b3ull;
    }
    return h;
}

WsView view_of(const dws_plan *p, void *ws) {
    unsigned char *base = static_cast<unsigned char *>(ws);
    WsView v;
    v.hdr = reinterpret_cast<WsHeader *>(base);
    v.numel = reinterpret_cast<const long long *>(base + p->layout.numel_off);
    v.first_tile = reinterpret_cast<const long long *>(base + p->layout.first_tile_off);
    v.tile_tensor = reinterpret_cast<const int *>(base + p->layout.tile_tensor_off);
    v.tile_status = reinterpret_cast<unsigned long long *>(base + p->layout.tile_status_off);
    v.tile_desc = reinterpret_cast<dws::TileDesc *>(base + p->layout.tile_desc_off);
    v.num_tiles = p->ntiles;
    v.num_tensors = p->T;
    v.fingerprint = p->fingerprint;
    return v;
}

dws_status_t check_ws(const dws_plan *p, const void *ws, size_t ws_bytes) {
    if (p == nullptr || ws == nullptr) return DWS_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DWS_ERR_WORKSPACE;
    if (ws_bytes < p->layout.total) return DWS_ERR_WORKSPACE;
    return DWS_OK;
}

dws_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? DWS_OK : DWS_ERR_CUDA; }

// DWS_CHAIN_AUTO's choice, from what the host knows (the entry counts): the
// merge moves every touched tile whole, the scatter only the touched 32-byte
// sectors, each read and written back by L2.  With the deltas' union covering
// a fraction u of the elements, about 1 - (1 - u)^16 of the sectors are
// touched; above one half the merge moves fewer bytes, or about as many at a
// better rate (whole-tile bulk copies against partial-sector writes).
// The scatter moves only the touched sectors and was the faster mode on
// every chain measured, dense or clustered.
int32_t chain_auto_mode() { return DWS_CHAIN_SCATTER; }

dws_status_t encode_common(const dws_plan_t *plan, const void *const *old_ptrs,
                           const void *const *new_ptrs, int64_t *offsets, int32_t *indices,
                           uint16_t *values, int64_t capacity, void *workspace,
                           size_t workspace_bytes, dws_stream_t stream, bool compact,
                           int64_t wait_limit_ns, int64_t withhold, int64_t *indices64 = nullptr,
                           const int64_t *index_base = nullptr, uint64_t *hashes = nullptr) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (old_ptrs == nullptr || new_ptrs == nullptr || offsets == nullptr) return DWS_ERR_INVALID;
    if (compact) {
        if (capacity < 0) return DWS_ERR_INVALID;
        if (capacity > 0 && ((indices == nullptr && indices64 == nullptr) || values == nullptr))
            return DWS_ERR_INVALID;
    }
    const WsView v = view_of(plan, workspace);
    return from_cuda(dws::launch_encode(
        v, reinterpret_cast<const uint16_t *const *>(old_ptrs),
        reinterpret_cast<const uint16_t *const *>(new_ptrs), reinterpret_cast<long long *>(offsets),
        reinterpret_cast<int *>(indices), values, compact ? capacity : 0, compact,
        wait_limit_ns, withhold, reinterpret_cast<cudaStream_t>(stream),
        reinterpret_cast<long long *>(indices64), reinterpret_cast<const long long *>(index_base),
        reinterpret_cast<unsigned long long *>(hashes)));
}

}  // namespace

extern "C" {

dws_status_t dws_plan_create(const int64_t *numels, int32_t num_tensors, int32_t elem_size,
                             dws_plan_t **plan_out) {
    if (plan_out == nullptr) return DWS_ERR_INVALID;
    *plan_out = nullptr;
    if (numels == nullptr || num_tensors <= 0) return DWS_ERR_INVALID;
    if (elem_size != 2) return DWS_ERR_UNSUPPORTED;
    int64_t N = 0, ntiles = 0;
    for (int32_t t = 0; t < num_tensors; ++t) {
        const int64_t n = numels[t];
        if (n < 0 || n > INT32_MAX) return DWS_ERR_INVALID;
        N += n;
        ntiles += (n == 0) ? 1 : (n + dws::kTileElems - 1) / dws::kTileElems;
    }
    dws_plan *p = new (std::nothrow) dws_plan;
    if (p == nullptr) return DWS_ERR_INVALID;
    p->T = num_tensors;
    p->N = N;
    p->ntiles = ntiles;
    p->layout = dws::ws_layout(num_tensors, ntiles);

    uint64_t h = 0xcbf29ce484222325ull;
    h = fnv1a(h, static_cast<uint64_t>(num_tensors));
    for (int32_t t = 0; t < num_tensors; ++t) h = fnv1a(h, static_cast<uint64_t>(numels[t]));
    p->fingerprint = h;

    // Static image: header, numel[T], first_tile[T+1] at their layout offsets.
    const size_t image_bytes = p->layout.tile_tensor_off;
    try {
        p->image.assign(image_bytes, 0);
    } catch (...) {
        delete p;
        return DWS_ERR_INVALID;
    }
    WsHeader hdr;
    std::memset(&hdr, 0, sizeof hdr);
    hdr.magic = dws::kWsMagic;
    hdr.fingerprint = p->fingerprint;
    hdr.num_tiles = ntiles;
    hdr.num_tensors = num_tensors;
    std::memcpy(p->image.data(), &hdr, sizeof hdr);
    long long *numel_img = reinterpret_cast<long long *>(p->image.data() + p->layout.numel_off);
    long long *first_img = reinterpret_cast<long long *>(p->image.data() + p->layout.first_tile_off);
    long long acc = 0;
    for (int32_t t = 0; t < num_tensors; ++t) {
        numel_img[t] = numels[t];
        first_img[t] = acc;
        acc += (numels[t] == 0) ? 1 : (numels[t] + dws::kTileElems - 1) / dws::kTileElems;
    }
    first_img[num_tensors] = acc;
    *plan_out = p;
    return DWS_OK;
}

void dws_plan_destroy(dws_plan_t *plan) { delete plan; }

int32_t dws_plan_num_tensors(const dws_plan_t *plan) { return plan ? plan->T : 0; }
int64_t dws_plan_num_elements(const dws_plan_t *plan) { return plan ? plan->N : 0; }
int64_t dws_plan_num_tiles(const dws_plan_t *plan) { return plan ? plan->ntiles : 0; }
int64_t dws_tile_elems(void) { return dws::kTileElems; }

size_t dws_plan_workspace_bytes(const dws_plan_t *plan) { return plan ? plan->layout.total : 0; }

dws_status_t dws_plan_upload(const dws_plan_t *plan, void *workspace, size_t workspace_bytes,
                             dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(workspace, plan->image.data(), plan->image.size(),
                                    cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return DWS_ERR_CUDA;
    return from_cuda(dws::launch_fill_tile_map(view_of(plan, workspace), s));
}

dws_status_t dws_encode(const dws_plan_t *plan, const void *const *old_ptrs,
                        const void *const *new_ptrs, int64_t *offsets, int32_t *indices,
                        uint16_t *values, int64_t capacity, void *workspace,
                        size_t workspace_bytes, dws_stream_t stream) {
    return encode_common(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, workspace,
                         workspace_bytes, stream, true, 0, -1);
}

dws_status_t dws_encode_nnz(const dws_plan_t *plan, const void *const *old_ptrs,
                            const void *const *new_ptrs, int64_t *offsets, int32_t *indices,
                            uint16_t *values, int64_t capacity, int64_t *nnz_dev, int64_t *nnz_host,
                            void *workspace, size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = encode_common(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                                    workspace, workspace_bytes, stream, true, 0, -1);
    if (st != DWS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t *total = offsets + plan->T;
    cudaError_t e = cudaSuccess;
    if (nnz_dev != nullptr) e = cudaMemcpyAsync(nnz_dev, total, sizeof(int64_t), cudaMemcpyDefault, s);
    if (e == cudaSuccess && nnz_host != nullptr)
        e = cudaMemcpyAsync(nnz_host, total, sizeof(int64_t), cudaMemcpyDefault, s);
    return from_cuda(e);
}

dws_status_t dws_encode_ex(const dws_plan_t *plan, const void *const *old_ptrs,
                           const void *const *new_ptrs, int64_t *offsets, int32_t *indices,
                           uint16_t *values, int64_t capacity, void *workspace,
                           size_t workspace_bytes, dws_stream_t stream, int64_t wait_limit_ns,
                           int64_t debug_withhold_tile) {
    return encode_common(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, workspace,
                         workspace_bytes, stream, true, wait_limit_ns, debug_withhold_tile);
}

dws_status_t dws_encode_global(const dws_plan_t *plan, const void *const *old_ptrs,
                               const void *const *new_ptrs, const int64_t *index_base,
                               int64_t *offsets, int64_t *indices, uint16_t *values,
                               int64_t capacity, void *workspace, size_t workspace_bytes,
                               dws_stream_t stream) {
    if (index_base == nullptr) return DWS_ERR_INVALID;
    if (capacity > 0 && indices == nullptr) return DWS_ERR_INVALID;
    // With no capacity nothing is written: the plain kernel computes the offsets.
    return encode_common(plan, old_ptrs, new_ptrs, offsets, nullptr, values, capacity, workspace,
                         workspace_bytes, stream, true, 0, -1, capacity > 0 ? indices : nullptr,
                         index_base);
}

dws_status_t dws_encode_checksum(const dws_plan_t *plan, const void *const *old_ptrs,
                                 const void *const *new_ptrs, int64_t *offsets, int32_t *indices,
                                 uint16_t *values, int64_t capacity, uint64_t *hashes,
                                 uint64_t *checksum, void *workspace, size_t workspace_bytes,
                                 dws_stream_t stream) {
    if (hashes == nullptr) return DWS_ERR_INVALID;
    dws_status_t st = encode_common(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                                    workspace, workspace_bytes, stream, true, 0, -1, nullptr,
                                    nullptr, hashes);
    if (st != DWS_OK || checksum == nullptr) return st;
    return from_cuda(dws::launch_checksum_wire(reinterpret_cast<const unsigned long long *>(hashes),
                                               reinterpret_cast<unsigned long long *>(checksum),
                                               reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_count(const dws_plan_t *plan, const void *const *old_ptrs,
                       const void *const *new_ptrs, int64_t *offsets, void *workspace,
                       size_t workspace_bytes, dws_stream_t stream) {
    return encode_common(plan, old_ptrs, new_ptrs, offsets, nullptr, nullptr, 0, workspace,
                         workspace_bytes, stream, false, 0, -1);
}

dws_status_t dws_apply(const dws_plan_t *plan, void *const *snap_ptrs, const int64_t *offsets,
                       const int32_t *indices, const uint16_t *values, int64_t count,
                       void *workspace, size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (snap_ptrs == nullptr || offsets == nullptr || count < 0) return DWS_ERR_INVALID;
    if (count > 0 && (indices == nullptr || values == nullptr)) return DWS_ERR_INVALID;
    dws::DeltaRef d{reinterpret_cast<const long long *>(offsets),
                    reinterpret_cast<const int *>(indices), values, count};
    return from_cuda(dws::launch_apply(view_of(plan, workspace),
                                       reinterpret_cast<uint16_t *const *>(snap_ptrs), d,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_apply_chain(const dws_plan_t *plan, void *const *snap_ptrs,
                             const dws_delta_t *deltas, int32_t K, void *workspace,
                             size_t workspace_bytes, dws_stream_t stream) {
    return dws_apply_chain_ex(plan, snap_ptrs, deltas, K, DWS_CHAIN_AUTO, workspace,
                              workspace_bytes, stream);
}

dws_status_t dws_apply_chain_ex(const dws_plan_t *plan, void *const *snap_ptrs,
                                const dws_delta_t *deltas, int32_t K, int32_t mode,
                                void *workspace, size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (snap_ptrs == nullptr || deltas == nullptr || K < 1 || K > DWS_MAX_CHAIN)
        return DWS_ERR_INVALID;
    if (mode != DWS_CHAIN_AUTO && mode != DWS_CHAIN_TILE_MERGE && mode != DWS_CHAIN_SCATTER)
        return DWS_ERR_INVALID;
    dws::DeltaRef d[DWS_MAX_CHAIN];
    for (int32_t k = 0; k < K; ++k) {
        if (deltas[k].offsets == nullptr || deltas[k].count < 0) return DWS_ERR_INVALID;
        if (deltas[k].count > 0 && (deltas[k].indices == nullptr || deltas[k].values == nullptr))
            return DWS_ERR_INVALID;
        if ((reinterpret_cast<uintptr_t>(deltas[k].indices) & 3u) ||
            (reinterpret_cast<uintptr_t>(deltas[k].values) & 1u) ||
            (reinterpret_cast<uintptr_t>(deltas[k].offsets) & 7u))
            return DWS_ERR_INVALID;
        d[k] = dws::DeltaRef{reinterpret_cast<const long long *>(deltas[k].offsets),
                             reinterpret_cast<const int *>(deltas[k].indices), deltas[k].values,
                             deltas[k].count};
    }
    if (mode == DWS_CHAIN_AUTO) mode = chain_auto_mode();
    return from_cuda(dws::launch_apply_chain(view_of(plan, workspace),
                                             reinterpret_cast<uint16_t *const *>(snap_ptrs), d, K,
                                             mode == DWS_CHAIN_TILE_MERGE,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_merge_shards(const dws_plan_t *plan, int32_t num_ranks,
                              const int64_t *rank_offsets, const int64_t *rank_indices,
                              const uint16_t *rank_values, int64_t stride, int64_t *offsets,
                              int64_t *indices, uint16_t *values, int64_t capacity,
                              void *workspace, size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (num_ranks < 1 || num_ranks > 65535 || rank_offsets == nullptr || offsets == nullptr ||
        stride < 0 || capacity < 0)
        return DWS_ERR_INVALID;
    if (stride > 0 && (rank_indices == nullptr || rank_values == nullptr)) return DWS_ERR_INVALID;
    if (capacity > 0 && (indices == nullptr || values == nullptr)) return DWS_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(rank_indices) & 7u) || (reinterpret_cast<uintptr_t>(indices) & 7u) ||
        (reinterpret_cast<uintptr_t>(rank_values) & 1u) || (reinterpret_cast<uintptr_t>(values) & 1u))
        return DWS_ERR_INVALID;
    return from_cuda(dws::launch_merge_shards(
        view_of(plan, workspace), num_ranks, reinterpret_cast<const long long *>(rank_offsets),
        reinterpret_cast<const long long *>(rank_indices), rank_values, stride,
        reinterpret_cast<long long *>(offsets), reinterpret_cast<long long *>(indices), values,
        capacity, reinterpret_cast<cudaStream_t>(stream)));
}

// Byte positions are int32: every layer below 2^30 words (2^31 bytes).
static bool bytes_fit_int32(const dws_plan_t *plan) {
    const long long *numel = reinterpret_cast<const long long *>(plan->image.data() + plan->layout.numel_off);
    for (int32_t t = 0; t < plan->T; ++t)
        if (numel[t] >= (1LL << 30)) return false;
    return true;
}

dws_status_t dws_xor_bytes_from_words(const dws_plan_t *plan, const void *const *old_ptrs,
                                      const int64_t *word_offsets, const int32_t *word_indices,
                                      const uint16_t *word_values, int64_t word_count, int64_t *byte_offsets,
                                      int32_t *byte_positions, uint8_t *byte_values, int64_t capacity,
                                      void *workspace, size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (old_ptrs == nullptr || word_offsets == nullptr || byte_offsets == nullptr || word_count < 0 ||
        capacity < 0)
        return DWS_ERR_INVALID;
    if (word_count > 0 && (word_indices == nullptr || word_values == nullptr)) return DWS_ERR_INVALID;
    if (capacity > 0 && (byte_positions == nullptr || byte_values == nullptr)) return DWS_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(word_indices) & 3u) || (reinterpret_cast<uintptr_t>(word_values) & 1u) ||
        (reinterpret_cast<uintptr_t>(byte_positions) & 3u) || (reinterpret_cast<uintptr_t>(byte_offsets) & 7u) ||
        (reinterpret_cast<uintptr_t>(word_offsets) & 7u))
        return DWS_ERR_INVALID;
    if (!bytes_fit_int32(plan)) return DWS_ERR_INVALID;
    dws::DeltaRef d{reinterpret_cast<const long long *>(word_offsets), reinterpret_cast<const int *>(word_indices),
                    word_values, word_count};
    return from_cuda(dws::launch_xor_bytes_from_words(
        view_of(plan, workspace), reinterpret_cast<const uint16_t *const *>(old_ptrs), d, plan->N,
        reinterpret_cast<long long *>(byte_offsets), reinterpret_cast<int *>(byte_positions), byte_values,
        capacity, reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_apply_bytes(const dws_plan_t *plan, void *const *buf_ptrs, const int64_t *offsets,
                             const int32_t *positions, const uint8_t *values, int64_t count, void *workspace,
                             size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (buf_ptrs == nullptr || offsets == nullptr || count < 0) return DWS_ERR_INVALID;
    if (count > 0 && (positions == nullptr || values == nullptr)) return DWS_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(positions) & 3u) || (reinterpret_cast<uintptr_t>(offsets) & 7u))
        return DWS_ERR_INVALID;
    if (!bytes_fit_int32(plan)) return DWS_ERR_INVALID;
    return from_cuda(dws::launch_apply_bytes(view_of(plan, workspace), reinterpret_cast<uint8_t *const *>(buf_ptrs),
                                             reinterpret_cast<const long long *>(offsets),
                                             reinterpret_cast<const int *>(positions), values, count,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int32_t dws_pos_width(const dws_plan_t *plan, int32_t t) {
    if (plan == nullptr || t < 0 || t >= plan->T) return 0;
    const long long *numel =
        reinterpret_cast<const long long *>(plan->image.data() + plan->layout.numel_off);
    return numel[t] <= 65536 ? 2 : 4;
}

dws_status_t dws_pack_positions(const dws_plan_t *plan, const int64_t *offsets,
                                const int32_t *indices, int64_t count, uint8_t *positions,
                                int64_t pos_capacity, int64_t *pos_offsets, void *workspace,
                                size_t workspace_bytes, dws_stream_t stream) {
    dws_status_t st = check_ws(plan, workspace, workspace_bytes);
    if (st != DWS_OK) return st;
    if (offsets == nullptr || pos_offsets == nullptr || count < 0 || pos_capacity < 0)
        return DWS_ERR_INVALID;
    if (count > 0 && indices == nullptr) return DWS_ERR_INVALID;
    if (pos_capacity > 0 && (positions == nullptr || (reinterpret_cast<uintptr_t>(positions) & 1u)))
        return DWS_ERR_INVALID;
    dws::DeltaRef d{reinterpret_cast<const long long *>(offsets),
                    reinterpret_cast<const int *>(indices), nullptr, count};
    return from_cuda(dws::launch_pack_positions(view_of(plan, workspace), d, positions, pos_capacity,
                                                reinterpret_cast<long long *>(pos_offsets),
                                                reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_checksum(const uint8_t *positions, int64_t pos_bytes, const uint16_t *values,
                          int64_t nnz, uint64_t *hashes, uint64_t *checksum, dws_stream_t stream) {
    if (hashes == nullptr || pos_bytes < 0 || nnz < 0) return DWS_ERR_INVALID;
    if ((pos_bytes > 0 && positions == nullptr) || (nnz > 0 && values == nullptr))
        return DWS_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(values) & 1u) return DWS_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = dws::launch_checksum(positions, pos_bytes, values, nnz,
                                         reinterpret_cast<unsigned long long *>(hashes), s);
    if (e == cudaSuccess && checksum != nullptr)
        e = dws::launch_checksum_wire(reinterpret_cast<const unsigned long long *>(hashes),
                                      reinterpret_cast<unsigned long long *>(checksum), s);
    return from_cuda(e);
}

dws_status_t dws_xor_encode(const void *old_bytes, const void *new_bytes, void *mask,
                            int64_t nbytes, dws_stream_t stream) {
    if (nbytes < 0) return DWS_ERR_INVALID;
    if (nbytes == 0) return DWS_OK;
    if (old_bytes == nullptr || new_bytes == nullptr || mask == nullptr) return DWS_ERR_INVALID;
    return from_cuda(dws::launch_xor(static_cast<const uint8_t *>(old_bytes),
                                     static_cast<const uint8_t *>(new_bytes),
                                     static_cast<uint8_t *>(mask), nbytes,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_xor_apply(void *buf, const void *mask, int64_t nbytes, dws_stream_t stream) {
    if (nbytes < 0) return DWS_ERR_INVALID;
    if (nbytes == 0) return DWS_OK;
    if (buf == nullptr || mask == nullptr) return DWS_ERR_INVALID;
    return from_cuda(dws::launch_xor(static_cast<const uint8_t *>(buf),
                                     static_cast<const uint8_t *>(mask),
                                     static_cast<uint8_t *>(buf), nbytes,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

dws_status_t dws_xor_apply_layers(void *const *bufs, const void *const *masks,
                                  const int64_t *nbytes, int32_t L, void *staging0,
                                  void *staging1, int64_t staging_bytes,
                                  dws_stream_t apply_stream, dws_stream_t copy_stream) {
    if (bufs == nullptr || masks == nullptr || nbytes == nullptr || L < 0) return DWS_ERR_INVALID;
    if (staging0 == nullptr || staging1 == nullptr || staging_bytes <= 0) return DWS_ERR_INVALID;
    for (int32_t l = 0; l < L; ++l) {
        if (nbytes[l] < 0) return DWS_ERR_INVALID;
        if (nbytes[l] > 0 && (bufs[l] == nullptr || masks[l] == nullptr)) return DWS_ERR_INVALID;
    }
    if (L == 0) return DWS_OK;
    cudaStream_t as = reinterpret_cast<cudaStream_t>(apply_stream);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
    void *staging[2] = {staging0, staging1};

    cudaEvent_t start, copied[2], applied[2];
    cudaError_t e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
    if (e != cudaSuccess) return DWS_ERR_CUDA;
    int made = 0;
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
        e = cudaEventCreateWithFlags(&copied[b], cudaEventDisableTiming);
        if (e == cudaSuccess) {
            e = cudaEventCreateWithFlags(&applied[b], cudaEventDisableTiming);
            if (e == cudaSuccess) ++made;
            else cudaEventDestroy(copied[b]);
        }
    }
    // The copy stream starts after what is already queued on the apply stream.
    if (e == cudaSuccess) e = cudaEventRecord(start, as);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, start, 0);

    bool used[2] = {false, false};
    long long unit = 0;
    for (int32_t l = 0; l < L && e == cudaSuccess; ++l) {
        for (int64_t off = 0; off < nbytes[l] && e == cudaSuccess; off += staging_bytes) {
            const int64_t len = (nbytes[l] - off < staging_bytes) ? (nbytes[l] - off) : staging_bytes;
            const int b = static_cast<int>(unit & 1);
            // Staging buffer b is free once the apply that read it is done.
            if (used[b]) e = cudaStreamWaitEvent(cs, applied[b], 0);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(staging[b], static_cast<const uint8_t *>(masks[l]) + off,
                                    static_cast<size_t>(len), cudaMemcpyDefault, cs);
            if (e == cudaSuccess) e = cudaEventRecord(copied[b], cs);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(as, copied[b], 0);
            if (e == cudaSuccess)
                e = dws::launch_xor(static_cast<const uint8_t *>(bufs[l]) + off,
                                    static_cast<const uint8_t *>(staging[b]),
                                    static_cast<uint8_t *>(bufs[l]) + off, len, as);
            if (e == cudaSuccess) e = cudaEventRecord(applied[b], as);
            used[b] = true;
            ++unit;
        }
    }
    // Events are released once their pending work completes.
    cudaEventDestroy(start);
    for (int b = 0; b < made; ++b) {
        cudaEventDestroy(copied[b]);
        cudaEventDestroy(applied[b]);
    }
    return from_cuda(e);
}

dws_status_t dws_status(void *workspace, int64_t *detail, dws_stream_t stream) {
    if (workspace == nullptr) return DWS_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WsHeader *hdr = static_cast<WsHeader *>(workspace);
    struct {
        unsigned int status;
        unsigned int pad;
        long long detail;
    } host{};
    cudaError_t e = cudaMemcpyAsync(&host.status, &hdr->status, sizeof(unsigned int),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&host.detail, &hdr->detail, sizeof(long long), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return DWS_ERR_CUDA;
    if (detail) *detail = host.detail;
    if (host.status != 0u) {
        e = cudaMemsetAsync(&hdr->status, 0, sizeof(unsigned int), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(&hdr->detail, 0, sizeof(long long), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return DWS_ERR_CUDA;
    }
    return static_cast<dws_status_t>(host.status);
}

const char *dws_strerror(dws_status_t status) {
    switch (status) {
        case DWS_OK: return "ok";
        case DWS_ERR_INVALID: return "invalid argument";
        case DWS_ERR_UNSUPPORTED: return "unsupported element size";
        case DWS_ERR_CAPACITY: return "output capacity exceeded";
        case DWS_ERR_BAD_DELTA: return "bad delta (index out of range, not ascending, or bad offsets)";
        case DWS_ERR_TIMEOUT: return "bounded wait ran out";
        case DWS_ERR_CUDA: return "CUDA runtime error";
        case DWS_ERR_WORKSPACE: return "workspace too small or not prepared for this plan";
    }
    return "unknown status";
}

dws_status_t dws_device_memory(int32_t device, int32_t *clock_khz, int32_t *bus_bits) {
    if (clock_khz == nullptr || bus_bits == nullptr) return DWS_ERR_INVALID;
    int khz = 0, bits = 0;
    cudaError_t e = cudaDeviceGetAttribute(&khz, cudaDevAttrMemoryClockRate, device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&bits, cudaDevAttrGlobalMemoryBusWidth, device);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return DWS_ERR_CUDA;
    }
    *clock_khz = khz;
    *bus_bits = bits;
    return DWS_OK;
}

uint64_t dws_launch_count(void) { return dws::g_launches.load(std::memory_order_relaxed); }

const char *dws_version(void) { return "libdws 0.1 sm_100a"; }

}  // extern "C"
