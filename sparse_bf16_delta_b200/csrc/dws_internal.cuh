// dws_internal.cuh -- shared definitions of libdws's kernels and host code:
// the workspace layout, the device status word, and thin inline-PTX wrappers
// for the sm_100a features the kernels use (mbarrier transaction counts,
// 1-D bulk async copies between global and shared memory, L2 eviction
// hints, gpu-scope relaxed loads/stores, the global nanosecond timer).
//
// No cluster multicast is used anywhere in libdws: every bulk copy moves data
// between this GPU's global memory and the issuing CTA's own shared memory.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/dws.h"

namespace dws {

// ---------------------------------------------------------------------------
// Tiling shared by the encode scan and the chain replay: a tensor is cut into
// tiles of kTileElems elements (16 KiB of bf16 per snapshot); a tile never
// straddles two tensors and an empty tensor owns one empty tile.
// ---------------------------------------------------------------------------
constexpr int kTileElems = 8192;
constexpr int kTileShift = 13;
// Tile status words sit one per 32-byte sector (every fourth word): all
// look-backs read the newest tiles' words, and packing them densely puts
// those reads on a few L2 lines (and slices).
constexpr int kStatusStride = 4;
static_assert((1 << kTileShift) == kTileElems, "tile size must be a power of two");
// The chain replay handles up to kChainGroup deltas per pass over the
// snapshot; its tile index holds, per tile and delta of the pass, the first
// entry at or past the tile (mod 2^32), kChainGroup words per tile.
constexpr int kChainGroup = 16;

// ---------------------------------------------------------------------------
// Workspace layout (device memory owned by the caller)
//
//   [0, 256)          WsHeader
//   numel             int64[T]           tensor sizes          (static)
//   first_tile        int64[T+1]         first tile of tensor  (static)
//   tile_tensor       int32[ntiles]      tensor of each tile   (static)
//   tile_status       uint64[ntiles * kStatusStride]  encode scan state (per call)
//   tile_desc         TileDesc[ntiles]   encode tile pointers  (per call)
//
// The chain replay's tile index, uint32[(ntiles + 1) * kChainGroup] (per
// call), overlays tile_status and tile_desc: 64 bytes per tile, the two
// regions' size, plus one more row that the total leaves room for.
//
// Every region starts on a 256-byte boundary.  The static regions are written
// by dws_plan_upload; the header's magic + fingerprint tie the workspace to
// the plan that wrote it.
// ---------------------------------------------------------------------------
constexpr unsigned long long kWsMagic = 0x3130305357534457ull;  // "DWSWS001"

// Two 128-byte lines.  The ticket counter, hit by every producer's atomic,
// has the second line to itself: waiting warps poll `abort`, and sharing a
// line (let alone a sector) with the counter would queue those reads behind
// the atomics at the L2, slowing the tickets in turn.
struct WsHeader {
    unsigned long long magic;        // 0
    unsigned long long fingerprint;  // 8
    long long num_tiles;             // 16
    int num_tensors;                 // 24
    unsigned int status;             // 28  first device error (dws_status_t), 0 = none
    long long detail;                // 32  detail of that error
    unsigned int abort;              // 40  encode: a bounded wait ran out, all waiters leave
    unsigned int delta_bad;          // 44  apply/chain: offsets of some delta failed validation
    unsigned char pad0[128 - 48];
    unsigned long long ticket;       // 128 encode: next tile ticket
    unsigned char pad1[256 - 136];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte block");

// Per-call description of an encode tile, written by the prepare pass so the
// encode kernel needs one 32-byte load per ticket.
struct TileDesc {
    const uint16_t *old_p;  // tile start in the old snapshot (null if count == 0)
    const uint16_t *new_p;  // tile start in the new snapshot
    int tensor;
    int local_start;  // first element of the tile within its tensor
    int count;        // elements in the tile (0 .. kTileElems)
    int bulk;         // leading elements that can move by bulk copy (multiple of 8)
};
static_assert(sizeof(TileDesc) == 32, "tile descriptor is 32 bytes");

struct WsLayout {
    size_t numel_off, first_tile_off, tile_tensor_off, tile_status_off, tile_desc_off, total;
};

inline size_t round_up256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int T, long long ntiles) {
    WsLayout L;
    L.numel_off = 256;
    L.first_tile_off = round_up256(L.numel_off + sizeof(long long) * size_t(T));
    L.tile_tensor_off = round_up256(L.first_tile_off + sizeof(long long) * size_t(T + 1));
    L.tile_status_off = round_up256(L.tile_tensor_off + sizeof(int) * size_t(ntiles));
    L.tile_desc_off = round_up256(L.tile_status_off +
                                  sizeof(unsigned long long) * size_t(ntiles) * kStatusStride);
    L.total = round_up256(L.tile_desc_off + sizeof(TileDesc) * size_t(ntiles));
    const size_t index_end =
        L.tile_status_off + sizeof(uint32_t) * size_t(kChainGroup) * size_t(ntiles + 1);
    if (L.total < round_up256(index_end)) L.total = round_up256(index_end);
    return L;
}

// Device view of a prepared workspace, passed by value to every kernel.
struct WsView {
    WsHeader *hdr;
    const long long *numel;
    const long long *first_tile;
    const int *tile_tensor;
    unsigned long long *tile_status;
    TileDesc *tile_desc;
    long long num_tiles;
    int num_tensors;
    unsigned long long fingerprint;
};

// Encode scan state per tile: 2 flag bits + a 62-bit count.
constexpr unsigned long long kFlagShift = 62;
constexpr unsigned long long kFlagAggregate = 1ull << kFlagShift;  // tile's own count
constexpr unsigned long long kFlagPrefix = 2ull << kFlagShift;     // inclusive prefix
constexpr unsigned long long kValueMask = (1ull << kFlagShift) - 1;

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ void record_error(WsHeader *hdr, unsigned int code, long long detail) {
    if (atomicCAS(&hdr->status, 0u, code) == 0u) {
        atomicExch(reinterpret_cast<unsigned long long *>(&hdr->detail),
                   static_cast<unsigned long long>(detail));
    }
}

// One thread per CTA checks that the workspace belongs to the plan of this
// launch; returns the verdict to every thread of the CTA.
__device__ __forceinline__ bool ws_matches(const WsView &ws) {
    __shared__ int ok;
    if (threadIdx.x == 0) {
        const WsHeader *h = ws.hdr;
        ok = (h->magic == kWsMagic && h->fingerprint == ws.fingerprint &&
              h->num_tiles == ws.num_tiles && h->num_tensors == ws.num_tensors);
        if (!ok) record_error(ws.hdr, DWS_ERR_WORKSPACE, 0);
    }
    __syncthreads();
    return ok != 0;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_gpu(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned int ld_relaxed_gpu_u32(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// L2 policy: data read once (snapshots, masks) is evicted first.
__device__ __forceinline__ unsigned long long l2_evict_first_policy() {
    unsigned long long pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// --- mbarrier (shared::cta) -------------------------------------------------
__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of `bar` to complete.  Bulk copies of valid memory
// always complete; the limit only keeps a broken invariant from spinning
// forever.  Returns false if the limit was reached.
__device__ __forceinline__ bool mbar_wait(unsigned long long *bar, uint32_t parity,
                                          unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// try_wait that lets the hardware suspend the thread for up to `hint_ns`
// while the phase is incomplete (instead of returning at once).
__device__ __forceinline__ bool mbar_try_wait_hint(unsigned long long *bar, uint32_t parity,
                                                   uint32_t hint_ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// mbar_wait for threads that may wait long: each test suspends the thread
// in hardware for up to a microsecond, leaving the issue slots to the warps
// that work.
__device__ __forceinline__ bool mbar_wait_sleepy(unsigned long long *bar, uint32_t parity,
                                                 unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait_hint(bar, parity, 1000u)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// --- 1-D bulk async copies (no tensor map, no multicast) --------------------
// global -> this CTA's shared memory, completion counted on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                          unsigned long long *bar, unsigned long long policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// this CTA's shared memory -> global, tracked by the issuing thread's bulk group.
__device__ __forceinline__ void bulk_store(void *gmem_dst, const void *smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
                 "r"(smem_addr(smem_src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// The issuing thread's committed bulk stores have finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// All but the n most recently committed bulk-store groups of the issuing
// thread have finished READING shared memory (n > 7 waits for all).
__device__ __forceinline__ void bulk_wait_read_n(int n) {
    switch (n) {
        case 1: asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.bulk.wait_group.read 5;" ::: "memory"); break;
        case 6: asm volatile("cp.async.bulk.wait_group.read 6;" ::: "memory"); break;
        case 7: asm volatile("cp.async.bulk.wait_group.read 7;" ::: "memory"); break;
        default: asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); break;
    }
}

// The issuing thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (a later bulk store reads them).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --- named barriers and CTA-scope release/acquire on shared memory -----------
// Barrier `id` among `count` threads (whole warps) of the CTA.
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier `id` among `count` threads returning the AND of `pred` over them.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void st_release_cta(int *p, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_cta(const int *p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}

// --- cache-hinted global accesses -------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream_v4(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_stream_v2(void *p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void st_stream_v2u64(void *p, unsigned long long a, unsigned long long b) {
    asm volatile("st.global.cs.v2.u64 [%0], {%1,%2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

__device__ __forceinline__ void st_stream_u64(void *p, unsigned long long v) {
    asm volatile("st.global.cs.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_stream_u32(void *p, uint32_t v) {
    asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_stream_u16(void *p, uint16_t v) {
    asm volatile("st.global.cs.u16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

// Tensor of delta entry j (a delta's offsets are non-decreasing).
// Largest t in [lo, hi] with offsets[t] <= j (offsets validated non-decreasing).
__device__ __forceinline__ int tensor_of_entry(const long long *offsets, int lo, int hi,
                                               long long j) {
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Warp-cooperative: the largest t in [0, T-1] with offsets[t] <= j (offsets
// non-decreasing, offsets[0] = 0 <= j).  Each round probes 32 evenly spaced
// tensors, so T = 291 takes two dependent loads and T = 12000 three.
__device__ __forceinline__ int warp_tensor_of_entry(const long long *offsets, int T, long long j) {
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = T - 1;  // the answer lies in [lo, hi]
    while (true) {
        const int span = hi - lo + 1;
        const int step = (span + 31) / 32;
        const int t = lo + lane * step;
        const bool le = (t <= hi) && (__ldg(offsets + t) <= j);
        const unsigned int b = __ballot_sync(0xffffffffu, le);  // a prefix of lanes; lane 0 set
        const int c = __popc(b);
        if (step == 1) return lo + c - 1;
        const int nlo = lo + (c - 1) * step;
        const int nhi = lo + c * step - 1;
        lo = nlo;
        hi = nhi < hi ? nhi : hi;
    }
}

// The double equal to a bf16 value, as bits: sign, exponent rebased from
// 127 to 1023, mantissa moved up; subnormals normalised; infinities kept;
// NaNs quieted (bit 51 set) with sign and payload kept.
__device__ __forceinline__ unsigned long long bf16_to_f64_bits(uint32_t b) {
    const unsigned long long sign = static_cast<unsigned long long>(b >> 15) << 63;
    const uint32_t e = (b >> 7) & 0xffu;
    const uint32_t m = b & 0x7fu;
    if (e == 0xffu) {
        const unsigned long long q = m ? ((1ull << 51) | (static_cast<unsigned long long>(m) << 45)) : 0ull;
        return sign | (0x7ffull << 52) | q;
    }
    if (e == 0u) {
        if (m == 0u) return sign;
        const int top = 31 - __clz(m);  // m = 2^top + rest, value = m * 2^-133
        const unsigned long long frac = static_cast<unsigned long long>(m - (1u << top)) << (52 - top);
        return sign | (static_cast<unsigned long long>(top + 1023 - 133) << 52) | frac;
    }
    return sign | (static_cast<unsigned long long>(e - 127 + 1023) << 52) |
           (static_cast<unsigned long long>(m) << 45);
}

// XOR of the bytes of a position stored in `width` (2 or 4) little-endian
// bytes: its contribution to the hash of a positions block.
__device__ __forceinline__ unsigned long long pos_bytes_xor(uint32_t pos, int width) {
    uint32_t x = pos ^ (pos >> 8);
    if (width == 4) x ^= (pos >> 16) ^ (pos >> 24);
    return x & 0xffu;
}

#endif  // __CUDACC__

// ---------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files, called by the C ABI)
// ---------------------------------------------------------------------------
struct DeviceInfo {
    int sm_count;
    int encode_ctas_per_sm;
    long long l2_bytes;
};

// Per-device constants and one-time kernel attribute setup (thread-safe).
cudaError_t device_info(DeviceInfo *out);

// Count one kernel launch (dws_launch_count); returns cudaGetLastError().
cudaError_t launched();

cudaError_t launch_fill_tile_map(const WsView &ws, cudaStream_t s);
cudaError_t launch_encode(const WsView &ws, const uint16_t *const *old_ptrs,
                          const uint16_t *const *new_ptrs, long long *offsets, int *indices,
                          uint16_t *values, long long capacity, bool compact,
                          long long wait_limit_ns, long long withhold_tile, cudaStream_t s,
                          long long *indices64 = nullptr, const long long *index_base = nullptr,
                          unsigned long long *hashes = nullptr);

struct DeltaRef {
    const long long *offsets;
    const int *indices;
    const uint16_t *values;
    long long count;
};

// Clears the workspace's delta flag (set by a failed validation) on the stream.
cudaError_t launch_delta_flag_clear(const WsView &ws, cudaStream_t s);
cudaError_t launch_delta_check(const WsView &ws, const DeltaRef *deltas, int K, cudaStream_t s);
// Rank 0's merge of gathered shard deltas (dws_merge_shards).
cudaError_t launch_merge_shards(const WsView &ws, int R, const long long *rank_offsets,
                                const long long *rank_indices, const uint16_t *rank_values,
                                long long stride, long long *offsets, long long *indices,
                                uint16_t *values, long long capacity, cudaStream_t s);
cudaError_t launch_apply(const WsView &ws, uint16_t *const *snap_ptrs, const DeltaRef &d,
                         cudaStream_t s);
// Chain replay (chain.cu): validation and tile index of every delta, then
// one pass per group of up to kChainGroup deltas, by tile merge (merge =
// true) or by reverse-order scatter.  Nothing is written unless every delta
// passes validation.
cudaError_t launch_apply_chain(const WsView &ws, uint16_t *const *snap_ptrs,
                               const DeltaRef *deltas, int K, bool merge, cudaStream_t s);

// The byte-granular sparse XOR delta from a word delta of the same layers
// (xorbytes.cu); plan_elems: the plan's total elements.
cudaError_t launch_xor_bytes_from_words(const WsView &ws, const uint16_t *const *old_ptrs, const DeltaRef &d,
                                        long long plan_elems, long long *byte_offsets, int *positions,
                                        uint8_t *values, long long capacity, cudaStream_t s);
cudaError_t launch_apply_bytes(const WsView &ws, uint8_t *const *buf_ptrs, const long long *offsets,
                               const int *positions, const uint8_t *values, long long count, cudaStream_t s);

cudaError_t launch_pack_positions(const WsView &ws, const DeltaRef &d, uint8_t *positions,
                                  long long pos_capacity, long long *pos_offsets, cudaStream_t s);
cudaError_t launch_checksum(const uint8_t *positions, long long nbytes, const uint16_t *values,
                            long long nval, unsigned long long *out, cudaStream_t s);
// wire[0..1] = hashes[0] ^ (hashes[1] << 1) as a 128-bit little-endian integer.
cudaError_t launch_checksum_wire(const unsigned long long *hashes, unsigned long long *wire,
                                 cudaStream_t s);

cudaError_t launch_xor(const uint8_t *a, const uint8_t *b, uint8_t *out, long long nbytes,
                       cudaStream_t s);

// The plan's tensor count and per-tensor element counts (host memory owned by
// the plan).  False for a null plan.
bool plan_numels(const dws_plan_t *plan, int32_t *num_tensors, const long long **numels);

}  // namespace dws
