// apply.cu -- receiver side: scatter one delta, or replay a chain of deltas
// onto an anchor, in place.
//
// What it computes ("Delta Weight Sync in TRL" §4.3 receive_weights): for
// each tensor t and entry j of its segment, snap_t[indices[j]] = values[j];
// for a chain (§4.1: anchor every N syncs, a new replica replays the deltas
// after the latest anchor) the deltas in order, the later one winning.
//
// dws_apply -- one delta, direct scatter.  Each CTA takes 2048 consecutive
//   entries (coalesced index/value reads) and, before its one barrier, has
//   them, the workspace header and two warp-cooperative searches for its
//   first and last tensor in flight together; then it range- and
//   order-checks every index and stores the 2-byte values.  DRAM traffic is
//   the touched 32-byte sectors (read-modify-write in L2) plus 6 bytes per
//   entry, which is less than streaming the snapshot through at the
//   densities the workloads have.
//
// dws_apply_chain -- K deltas, one launch, two modes:
//   scatter (the default; chain_scatter_kernel): one CTA per SM owns whole
//   windows of 32 tiles; per window the deltas are replayed from the last to
//   the first, an element being stored only if its written-bit is clear, so
//   every element is written once, by the latest delta that touches it, and
//   untouched sectors are not moved at all.  Per delta, a window's entries
//   are one contiguous stretch, streamed by all warps in 32-entry chunks.
//   tile merge (chain_kernel): each CTA owns a contiguous range of snapshot
//   tiles; per tile a 1-D bulk async copy brings the tile into shared memory
//   while the CTA tags every delta's entries for it into a shared array with
//   atomicMax on ((k+1) << 16 | value) (the latest delta wins regardless of
//   thread order); the merged tile goes back with a bulk store.  It moves
//   the whole snapshot even where the deltas touch nothing.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr unsigned long long kLoadWaitLimitNs = 4000000000ull;  // 4 s

// ---------------------------------------------------------------------------
// Validation of the deltas' offsets (one CTA per delta), before any write.
// ---------------------------------------------------------------------------
struct CheckParams {
    WsView ws;
    DeltaRef d[DWS_MAX_CHAIN];
    int K;
};

__global__ void delta_check_kernel(CheckParams p) {
    if (!ws_matches(p.ws)) return;
    const DeltaRef d = p.d[blockIdx.x];
    const int T = p.ws.num_tensors;
    int bad = 0;
    if (threadIdx.x == 0) {
        bad |= (d.offsets[0] != 0);
        bad |= (d.offsets[T] > d.count);
    }
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        bad |= (d.offsets[t] > d.offsets[t + 1]);
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        if (bad) {
            atomicOr(&p.ws.hdr->delta_bad, 1u);
            record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, -1 - static_cast<long long>(blockIdx.x));
        }
    }
}

__global__ void delta_flag_clear_kernel(WsView ws) { ws.hdr->delta_bad = 0u; }

// ---------------------------------------------------------------------------
// Single delta: direct scatter
// ---------------------------------------------------------------------------
constexpr int kApplyThreads = 256;
constexpr int kApplyPerThread = 8;
constexpr int kApplyEntries = kApplyThreads * kApplyPerThread;

struct ApplyParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    DeltaRef d;
};

__global__ void __launch_bounds__(kApplyThreads) apply_kernel(ApplyParams p) {
    __shared__ int s_t[2];
    __shared__ int s_go;
    __shared__ long long s_end;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = p.ws.num_tensors;
    const long long base = static_cast<long long>(blockIdx.x) * kApplyEntries;
    const long long cap = p.d.count;  // entries the arrays hold
    if (base >= cap) return;          // uniform

    // Everything below is read before any check, so that the latencies
    // overlap: the entries (the caller's arrays, bounded by count), the
    // workspace header and the delta's offsets.  Nothing is written until
    // the checks have passed.
    int idx[kApplyPerThread];
    uint16_t val[kApplyPerThread];
#pragma unroll
    for (int r = 0; r < kApplyPerThread; ++r) {
        const long long j = base + tid + r * kApplyThreads;
        if (j < cap) {
            idx[r] = __ldg(p.d.indices + j);
            val[r] = __ldg(p.d.values + j);
        }
    }
    if (warp < 2) {  // tensors of the block's first and last entries
        const long long last = (base + kApplyEntries < cap ? base + kApplyEntries : cap) - 1;
        const int t = warp_tensor_of_entry(p.d.offsets, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    if (tid == 64) {
        const WsHeader *h = p.ws.hdr;
        const bool ok = (h->magic == kWsMagic && h->fingerprint == p.ws.fingerprint &&
                         h->num_tiles == p.ws.num_tiles && h->num_tensors == T);
        if (!ok) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, 0);
        const long long nnz = p.d.offsets[T];
        const long long total = nnz < cap ? nnz : cap;
        const long long end = (base + kApplyEntries < total) ? base + kApplyEntries : total;
        s_end = end;
        s_go = ok && (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) == 0u) && base < end;
    }
    __syncthreads();
    if (!s_go) return;
    const long long end = s_end;
    const int t0 = s_t[0], t1 = s_t[1];

#pragma unroll
    for (int r = 0; r < kApplyPerThread; ++r) {
        const long long j = base + tid + r * kApplyThreads;
        // entry j - 1 is the previous lane's (lane 0: read it)
        int prev = __shfl_up_sync(0xffffffffu, idx[r], 1);
        if (j >= end) continue;
        const int t = (t0 == t1) ? t0 : tensor_of_entry(p.d.offsets, t0, t1, j);
        const long long n = p.ws.numel[t];
        const long long seg = p.d.offsets[t];
        const int i = idx[r];
        bool ok = (i >= 0) && (static_cast<long long>(i) < n);
        if (ok && j > seg) {
            if (lane == 0) prev = __ldg(p.d.indices + j - 1);
            ok = prev < i;
        }
        uint16_t *dst = p.snap_ptrs[t];
        if (ok && dst != nullptr && (reinterpret_cast<uintptr_t>(dst) & 1u) == 0) {
            dst[i] = val[r];
        } else {
            record_error(p.ws.hdr, ok ? DWS_ERR_INVALID : DWS_ERR_BAD_DELTA, j);
        }
    }
}

// ---------------------------------------------------------------------------
// Chain replay: tile merge
// ---------------------------------------------------------------------------
constexpr int kChainThreads = 256;
constexpr int kChainMaxSlots = 4096;  // K * block_len entries read per round
constexpr int kChainSlotsPerThread = kChainMaxSlots / kChainThreads;

struct ChainParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    long long tiles_per_cta;
    int K;
    int block_len;  // entries read per delta per round (multiple of 32)
    DeltaRef d[DWS_MAX_CHAIN];
};

// A unit: up to kChainUnitTiles consecutive plan tiles of one tensor.
struct UnitMeta {
    uint16_t *ptr;   // unit start in the snapshot
    long long next;  // first plan tile after the unit
    int tensor;
    int local_start;
    int count;
    int bulk;  // leading elements moved by bulk copies (multiple of 8)
};

struct ChainSmem {
    uint16_t tile[2][kChainUnitElems];
    uint32_t tag[kChainUnitElems];
    long long cur[DWS_MAX_CHAIN];
    long long end[DWS_MAX_CHAIN];
    long long seg[DWS_MAX_CHAIN];             // first entry of the current tensor's segment
    unsigned long long stop[DWS_MAX_CHAIN];   // first entry of this round not taken
    int active[DWS_MAX_CHAIN];
    unsigned long long bar[2];
    UnitMeta meta[2];
};

// Thread 0: describe the unit starting at plan tile i (ending before `te`)
// and start its load into buffer b.
__device__ void chain_issue(const ChainParams &p, ChainSmem &sm, long long i, long long te, int b,
                            unsigned long long policy) {
    UnitMeta m;
    m.ptr = nullptr;
    m.next = i + 1;
    m.tensor = 0;
    m.local_start = 0;
    m.count = 0;
    m.bulk = 0;
    const int t = p.ws.tile_tensor[i];
    if (t >= 0 && t < p.ws.num_tensors) {
        const long long first = p.ws.first_tile[t];
        long long j = p.ws.first_tile[t + 1];
        if (j > i + kChainUnitTiles) j = i + kChainUnitTiles;
        if (j > te) j = te;
        const long long ls = (i - first) << kTileShift;
        const long long n = p.ws.numel[t];
        if (ls >= 0 && ls <= n && j > i) {
            const long long rest = n - ls;
            const long long span = (j - i) << kTileShift;
            m.next = j;
            m.tensor = t;
            m.local_start = static_cast<int>(ls);
            m.count = static_cast<int>(rest < span ? rest : span);
            uint16_t *sp = p.snap_ptrs[t];
            const uintptr_t ua = reinterpret_cast<uintptr_t>(sp);
            if (m.count > 0 && (sp == nullptr || (ua & 1u))) {
                record_error(p.ws.hdr, DWS_ERR_INVALID, t);
                m.count = 0;
            } else if (m.count > 0) {
                m.ptr = sp + ls;
                m.bulk = (ua & 15u) == 0 ? (m.count & ~7) : 0;
            }
        } else {
            record_error(p.ws.hdr, DWS_ERR_WORKSPACE, i);
        }
    } else {
        record_error(p.ws.hdr, DWS_ERR_WORKSPACE, i);
    }
    mbar_arrive_expect_tx(&sm.bar[b], static_cast<uint32_t>(m.bulk) * 2u);
    if (m.bulk > 0) bulk_load(sm.tile[b], m.ptr, static_cast<uint32_t>(m.bulk) * 2u, &sm.bar[b], policy);
    sm.meta[b] = m;
}

// Warp-cooperative lower bound: first position in [lo, hi) whose index is
// >= key (indices ascending within the segment).
__device__ long long warp_lower_bound(const int *indices, long long lo, long long hi, int key) {
    const int lane = threadIdx.x & 31;
    while (hi - lo > 32) {
        const long long step = (hi - lo) / 32;
        const long long pos = lo + lane * step;
        const int v = indices[pos];
        const unsigned int below = __ballot_sync(0xffffffffu, v < key);
        const int c = __popc(below);
        if (c == 0) return lo;  // indices[lo] >= key
        const long long new_lo = lo + (c - 1) * step + 1;
        if (c < 32) hi = lo + c * step;
        lo = new_lo;
    }
    const long long pos = lo + lane;
    const int v = (pos < hi) ? indices[pos] : 0x7fffffff;
    const unsigned int below = __ballot_sync(0xffffffffu, v < key);
    return lo + __popc(below);
}

__global__ void __launch_bounds__(kChainThreads, 3) chain_kernel(ChainParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ChainSmem &sm = *reinterpret_cast<ChainSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    constexpr int kWarps = kChainThreads / 32;

    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;

    const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_cta;
    long long te = tb + p.tiles_per_cta;
    if (te > p.ws.num_tiles) te = p.ws.num_tiles;
    if (tb >= te) return;

    unsigned long long policy = 0;
    for (int e = tid; e < kChainUnitElems; e += kChainThreads) sm.tag[e] = 0u;
    if (tid == 0) {
        policy = l2_evict_first_policy();
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        mbar_fence_init();
        chain_issue(p, sm, tb, te, 0, policy);
    }
    __syncthreads();

    // Cursors at the CTA's first unit: one binary search per delta.
    {
        const UnitMeta m0 = sm.meta[0];
        for (int k = warp; k < p.K; k += kWarps) {
            const DeltaRef d = p.d[k];
            const long long lo = d.offsets[m0.tensor];
            const long long hi = d.offsets[m0.tensor + 1];
            // At a tensor's first tile start at the segment head, so that a
            // negative index is seen (and flagged) rather than skipped.
            const long long c = (m0.local_start == 0)
                                    ? lo
                                    : warp_lower_bound(d.indices, lo, hi, m0.local_start);
            if (lane == 0) {
                sm.cur[k] = c;
                sm.end[k] = hi;
                sm.seg[k] = lo;
                sm.stop[k] = ~0ull;
            }
        }
    }
    __syncthreads();

    const int L = p.block_len;
    const int slots = p.K * L;
    uint32_t phase_bits = 0;
    int b = 0;
    bool first_unit = true;
    for (long long i = tb; i < te;) {
        const UnitMeta m = sm.meta[b];
        if (tid == 0 && m.next < te) {
            bulk_wait_read_all();  // the store from the other buffer has read it
            chain_issue(p, sm, m.next, te, b ^ 1, policy);
        }
        const int ls = m.local_start;

        // New tensor inside the CTA's range: the previous tensor's entries
        // must all have been consumed (else some index was >= numel).
        if (!first_unit && ls == 0) {
            if (tid < p.K) {
                const DeltaRef d = p.d[tid];
                if (sm.cur[tid] != sm.end[tid]) record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, sm.cur[tid]);
                sm.cur[tid] = d.offsets[m.tensor];
                sm.seg[tid] = sm.cur[tid];
                sm.end[tid] = d.offsets[m.tensor + 1];
            }
        }
        if (tid < p.K) sm.active[tid] = (sm.cur[tid] < sm.end[tid]);
        __syncthreads();

        // ---- entry phase: tag this unit's entries of every delta ----------
        // Per round, L entries of every active delta from its cursor.  An
        // entry inside the unit is tagged unless it is not above the entry
        // before it in its tensor's segment; an entry below the unit is bad;
        // both are taken (consumed).  The first entry past the unit ends the
        // delta's stretch for this unit: the cursor moves to it.
        for (;;) {
            int idx[kChainSlotsPerThread];
            uint16_t val[kChainSlotsPerThread];
            int pidx[kChainSlotsPerThread];
            bool valid[kChainSlotsPerThread];
#pragma unroll
            for (int q = 0; q < kChainSlotsPerThread; ++q) {
                const int sidx = tid + q * kChainThreads;
                valid[q] = false;
                if (sidx < slots) {
                    const int k = sidx / L;
                    const long long j = sm.cur[k] + (sidx - k * L);
                    if (sm.active[k] && j < sm.end[k]) {
                        valid[q] = true;
                        idx[q] = __ldg(p.d[k].indices + j);
                        val[q] = __ldg(p.d[k].values + j);
                        if (lane == 0 && j > sm.seg[k]) pidx[q] = __ldg(p.d[k].indices + j - 1);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kChainSlotsPerThread; ++q) {
                const int sidx = tid + q * kChainThreads;
                if (q * kChainThreads >= slots) break;  // uniform across the CTA
                // 32 consecutive slots of a warp belong to one delta (L is a
                // multiple of 32) and hold consecutive entries.
                const int up = __shfl_up_sync(0xffffffffu, idx[q], 1);
                bool take = false;
                long long j = 0;
                if (valid[q]) {
                    const int k = sidx / L;
                    j = sm.cur[k] + (sidx - k * L);
                    const int prev = (lane == 0) ? pidx[q] : up;
                    const bool ordered = (j == sm.seg[k]) || (prev < idx[q]);
                    if (idx[q] < ls) {
                        // Below the unit (not ascending, or negative): bad.
                        record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, j);
                        take = true;
                    } else if (idx[q] - ls < m.count) {
                        if (ordered) {
                            const uint32_t key = (static_cast<uint32_t>(k + 1) << 16) | val[q];
                            atomicMax(&sm.tag[idx[q] - ls], key);
                        } else {
                            record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, j);
                        }
                        take = true;
                    }
                }
                const unsigned int left = __ballot_sync(0xffffffffu, valid[q] && !take);
                if (left != 0u && lane == __ffs(left) - 1)
                    atomicMin(&sm.stop[sidx / L], static_cast<unsigned long long>(j));
            }
            __syncthreads();
            int again = 0;
            if (tid < p.K) {
                const unsigned long long st = sm.stop[tid];
                sm.stop[tid] = ~0ull;
                if (sm.active[tid]) {
                    if (st != ~0ull) {
                        sm.cur[tid] = static_cast<long long>(st);
                    } else {
                        const long long nc = sm.cur[tid] + L;
                        sm.cur[tid] = nc < sm.end[tid] ? nc : sm.end[tid];
                        again = sm.cur[tid] < sm.end[tid];
                    }
                    sm.active[tid] = again;
                }
            }
            if (!__syncthreads_or(again)) break;
        }

        // ---- merge: tags over the snapshot unit ----------------------------
        const uint32_t parity = (phase_bits >> b) & 1u;
        phase_bits ^= (1u << b);
        const bool loaded = mbar_wait(&sm.bar[b], parity, kLoadWaitLimitNs);
        if (!__syncthreads_and(loaded)) {  // leave together, before any write
            if (tid == 0) record_error(p.ws.hdr, DWS_ERR_TIMEOUT, i);
            return;
        }
        int touched = 0;
        for (int c = tid; c * 8 < m.count; c += kChainThreads) {
            const int e0 = c * 8;
            uint4 t0 = *reinterpret_cast<const uint4 *>(&sm.tag[e0]);
            uint4 t1 = *reinterpret_cast<const uint4 *>(&sm.tag[e0 + 4]);
            const uint32_t any = t0.x | t0.y | t0.z | t0.w | t1.x | t1.y | t1.z | t1.w;
            if (any == 0u) continue;
            touched = 1;
            const uint32_t tg[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            *reinterpret_cast<uint4 *>(&sm.tag[e0]) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(&sm.tag[e0 + 4]) = make_uint4(0, 0, 0, 0);
            if (e0 + 8 <= m.bulk) {
                uint16_t *v = &sm.tile[b][e0];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (tg[q]) v[q] = static_cast<uint16_t>(tg[q] & 0xffffu);
            } else {
                // Outside the bulk-copied part: write straight to the snapshot.
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (tg[q] && e0 + q < m.count) m.ptr[e0 + q] = static_cast<uint16_t>(tg[q] & 0xffffu);
            }
        }
        if (m.bulk > 0) fence_proxy_async_smem();
        touched = __syncthreads_or(touched);
        if (tid == 0 && touched && m.bulk > 0) {
            bulk_store(m.ptr, sm.tile[b], static_cast<uint32_t>(m.bulk) * 2u);
            bulk_commit();
        }
        i = m.next;
        b ^= 1;
        first_unit = false;
    }

    // The CTA's range ends at the end of a tensor: all of its entries must
    // have been consumed.
    {
        const long long last = te - 1;
        const int t = p.ws.tile_tensor[last];
        const bool tensor_ends = (last + 1 == p.ws.num_tiles) || (p.ws.tile_tensor[last + 1] != t);
        if (tensor_ends && tid < p.K && sm.cur[tid] != sm.end[tid])
            record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, sm.cur[tid]);
    }
    if (tid == 0) bulk_wait_all();
}

// ---------------------------------------------------------------------------
// Chain replay: reverse-order scatter over windows, with a written-bitmap
// ---------------------------------------------------------------------------
// Each CTA owns a contiguous range of plan tiles and walks it in windows of
// kWinTiles tiles.  Per window the deltas are replayed from the LAST to the
// first: an entry is stored only if no later delta has stored that element
// (one bit per element of the window in shared memory), which leaves exactly
// what the forward replay leaves, and every element is written at most once.
// The snapshot is never read by the SM; partial 32-byte sectors are merged in
// L2.  Per delta, the window's entries are one contiguous stretch of the
// delta (entries are ordered by tensor, then index): the CTA's warps stream
// it in chunks of 32 entries, kScatDepth chunks in flight per warp, and the
// stretch ends at the first entry past the window, which is where the next
// window's stretch starts.
constexpr int kScatThreads = 1024;
constexpr int kScatWarps = kScatThreads / 32;
constexpr int kWinTiles = 32;
constexpr int kWinElems = kWinTiles * kTileElems;
constexpr int kScatDepth = 4;
constexpr long long kMaxStretch = 1LL << 30;  // entries one phase streams at most

struct ScatParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    long long tiles_per_cta;
    int K;
    DeltaRef d[DWS_MAX_CHAIN];
};

struct ScatSmem {
    uint32_t written[kWinElems / 32];
    long long cur[DWS_MAX_CHAIN];          // per delta: first entry not yet consumed
    long long base[kWinTiles];             // per window tensor: (first_tile - window start) * tile
    long long numel[kWinTiles];
    uint16_t *ptr[kWinTiles];
    long long offs[2][kWinTiles + 1];      // a delta's offsets of the window tensors (by phase parity)
    unsigned long long next[2];            // first entry past the window (min over warps)
};

__global__ void __launch_bounds__(kScatThreads, 1) chain_scatter_kernel(ScatParams p) {
    extern __shared__ __align__(128) unsigned char scat_smem_raw[];
    ScatSmem &sm = *reinterpret_cast<ScatSmem *>(scat_smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;

    const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_cta;
    long long te = tb + p.tiles_per_cta;
    if (te > p.ws.num_tiles) te = p.ws.num_tiles;
    if (tb >= te) return;

    // Cursors at the CTA's first tile: one warp-cooperative search per delta.
    {
        const int t0 = p.ws.tile_tensor[tb];
        const long long ls = (tb - p.ws.first_tile[t0]) << kTileShift;
        for (int k = warp; k < p.K; k += kScatWarps) {
            const DeltaRef d = p.d[k];
            const long long lo = d.offsets[t0];
            const long long hi = d.offsets[t0 + 1];
            // At a tensor's first tile start at the segment head, so that a
            // negative index is seen (and flagged) rather than skipped.
            const long long c = (ls == 0) ? lo : warp_lower_bound(d.indices, lo, hi, static_cast<int>(ls));
            if (lane == 0) sm.cur[k] = c;
        }
    }

    for (long long a = tb; a < te; a += kWinTiles) {
        const long long b = (a + kWinTiles < te) ? a + kWinTiles : te;
        const int win_words = static_cast<int>(b - a) * (kTileElems / 32);
        const int t_lo = p.ws.tile_tensor[a];
        const int nt = p.ws.tile_tensor[b - 1] - t_lo + 1;  // <= b - a: every tensor owns a tile
        if (t_lo < 0 || nt < 1 || nt > kWinTiles || t_lo + nt > p.ws.num_tensors) {
            if (tid == 0) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, a);
            return;  // uniform: every thread read the same table entries
        }
        __syncthreads();  // previous window (and the cursor set-up) complete
        for (int w = tid; w < win_words; w += kScatThreads) sm.written[w] = 0u;
        if (tid < nt) {
            const int t = t_lo + tid;
            const long long n = p.ws.numel[t];
            uint16_t *ptr = p.snap_ptrs[t];
            if (n > 0 && (ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 1u))) {
                record_error(p.ws.hdr, DWS_ERR_INVALID, t);
                ptr = nullptr;
            }
            sm.base[tid] = (p.ws.first_tile[t] - a) << kTileShift;
            sm.numel[tid] = n;
            sm.ptr[tid] = ptr;
        }
        const long long win_len = (b - a) << kTileShift;
        constexpr long long kStride = 32LL * kScatWarps;
        if (tid <= nt) sm.offs[(p.K - 1) & 1][tid] = p.d[p.K - 1].offsets[t_lo + tid];
        if (tid == 0) sm.next[(p.K - 1) & 1] = ~0ull;

        int ix[kScatDepth];
        uint16_t vx[kScatDepth];
        int px[kScatDepth];  // lane 0: the index of the entry before its chunk
        bool prefetched = false;  // the phase's first chunks already requested (uniform)
        for (int k = p.K - 1; k >= 0; --k) {
            const DeltaRef d = p.d[k];
            const int ph = k & 1;
            const long long *offs = sm.offs[ph];
            if (k == p.K - 1) __syncthreads();  // the window's set-up visible (later phases: below)
            const long long jmax = offs[nt];
            const long long j0 = sm.cur[k];
            // Positions relative to the stretch start, in 32 bits: a stretch
            // holds at most one window of valid entries (a delta's indices
            // are unique); one that runs longer (bad entries) is cut at
            // kMaxStretch and the next window goes on from there.
            const long long span = jmax - j0;
            const int n = static_cast<int>(span < kMaxStretch ? span : kMaxStretch);
            const int *pi = d.indices + j0;
            const uint16_t *pv = d.values + j0;
            int r = 32 * warp + lane;  // this lane's entry of the current chunk
            if (!prefetched) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (r + q * kStride < n) {
                        ix[q] = __ldg(pi + r + q * kStride);
                        vx[q] = __ldg(pv + r + q * kStride);
                        if (lane == 0 && j0 + r + q * kStride > 0) px[q] = __ldg(pi + r + q * kStride - 1);
                    }
                }
            }
            // The warp's current tensor (its chunks only move forward) and
            // that tensor's constants: segment (relative to j0, clamped to
            // [-1, n]), window offset, size, pointer.
            auto clamp_rel = [&](long long x) -> int {
                x -= j0;
                return static_cast<int>(x < -1 ? -1 : (x > n ? n : x));
            };
            int tw = 0;
            int seg_lo = clamp_rel(offs[0]), seg_hi = clamp_rel(offs[1]);
            int off_c = static_cast<int>(-sm.base[0]);  // window start - tensor start (elements)
            uint32_t numel_c = static_cast<uint32_t>(sm.numel[0]);
            uint16_t *ptr_c = sm.ptr[0];
            bool stop = false;
            for (;;) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    const int cs = r - lane;
                    if (cs >= n) {  // whole chunk past the stretch (uniform)
                        stop = true;
                        break;
                    }
                    const int idx = ix[q];
                    const uint16_t val = vx[q];
                    // the previous entry's index (lane 0: loaded with the chunk)
                    const int up = __shfl_up_sync(0xffffffffu, idx, 1);
                    const int prev = (lane == 0) ? px[q] : up;
                    if (r + kScatDepth * kStride < n) {
                        ix[q] = __ldg(pi + r + kScatDepth * kStride);
                        vx[q] = __ldg(pv + r + kScatDepth * kStride);
                        if (lane == 0) px[q] = __ldg(pi + r + kScatDepth * kStride - 1);
                    }
                    const bool valid = r < n;
                    if (cs >= seg_hi) {  // uniform: move to the chunk's first tensor
                        while (tw + 1 < nt && offs[tw + 1] <= j0 + cs) ++tw;
                        seg_lo = clamp_rel(offs[tw]);
                        seg_hi = clamp_rel(offs[tw + 1]);
                        off_c = static_cast<int>(-sm.base[tw]);
                        numel_c = static_cast<uint32_t>(sm.numel[tw]);
                        ptr_c = sm.ptr[tw];
                    }
                    const int cl = (cs + 31 < n) ? cs + 31 : n - 1;
                    // 0: nothing, 1: store, 2: bad entry (consumed), 3: past the window
                    int cls = 0;
                    uint32_t rel = 0;  // element within the window (when cls == 1)
                    uint16_t *dst = ptr_c;
                    if (cs >= seg_lo && cl < seg_hi) {
                        // Common case, all 32-bit: the chunk lies in one tensor.
                        // (off_c < numel <= 2^31 - 1; rel wraps for indices
                        // below the window, which `before` catches.)
                        // An entry not above the one before it in its
                        // tensor's segment is bad (as in dws_apply).
                        const bool ok = static_cast<uint32_t>(idx) < numel_c;
                        const bool before = idx < off_c;
                        const bool ordered = (r <= seg_lo) || (prev < idx);
                        rel = static_cast<uint32_t>(idx) - static_cast<uint32_t>(off_c);
                        if (valid)
                            cls = (!ok || before || !ordered)
                                      ? 2
                                      : (rel >= static_cast<uint32_t>(win_len) ? 3 : 1);
                    } else if (valid) {
                        // The chunk crosses a tensor boundary: per-lane tensor.
                        const long long j = j0 + r;
                        int tl = tw;
                        while (tl + 1 < nt && offs[tl + 1] <= j) ++tl;
                        if (j < offs[tl] || idx < 0 || static_cast<long long>(idx) >= sm.numel[tl] ||
                            (j > offs[tl] && prev >= idx)) {
                            cls = 2;
                        } else {
                            const long long e = sm.base[tl] + idx;
                            cls = (e >= win_len) ? 3 : (e < 0 ? 2 : 1);
                            rel = static_cast<uint32_t>(e);
                            dst = sm.ptr[tl];
                        }
                    }
                    const unsigned int past = __ballot_sync(0xffffffffu, cls == 3);
                    if (past != 0u) {
                        const int first = __ffs(past) - 1;
                        if (lane == first) atomicMin(&sm.next[ph], static_cast<unsigned long long>(j0 + r));
                        if (lane > first) cls = 0;
                        stop = true;
                    }
                    const bool ins = (cls == 1);
                    bool store = ins;
                    if (p.K > 1) {  // uniform: a single delta needs no written-bits
                        const uint32_t word = rel >> 5;
                        const uint32_t bit = 1u << (rel & 31u);
                        if (ins) store = (sm.written[word] & bit) == 0u;
                        // Mark this delta's elements: one OR per lane, or two
                        // for a run of 32 consecutive elements (a clustered
                        // change), where per-lane ORs would all hit one word.
                        const uint32_t r0 = __shfl_sync(0xffffffffu, rel, 0);
                        const uint32_t r31 = __shfl_sync(0xffffffffu, rel, 31);
                        bool marked = false;
                        if (r31 - r0 == 31u) {  // uniform; a run if all 32 ascend
                            const uint32_t prev = __shfl_up_sync(0xffffffffu, rel, 1);
                            const unsigned int run =
                                __ballot_sync(0xffffffffu, ins && (lane == 0 || rel > prev));
                            if (run == 0xffffffffu) {
                                if (lane == 0) atomicOr(&sm.written[r0 >> 5], ~0u << (r0 & 31u));
                                if (lane == 31 && (r31 & 31u) != 31u)
                                    atomicOr(&sm.written[r31 >> 5], (2u << (r31 & 31u)) - 1u);
                                marked = true;
                            }
                        }
                        if (!marked && ins) atomicOr(&sm.written[word], bit);
                    }
                    if (store) {
                        if (dst != nullptr) dst[idx] = val;
                    } else if (cls == 2) {
                        record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, j0 + r);
                    }
                    if (stop) break;
                    r += kStride;
                }
                if (stop) break;
            }
            // This warp is done with delta k.  While the others finish,
            // request the next (earlier) delta's offsets and first chunks:
            // its stretch starts at its cursor, and reading up to its count
            // stays inside its arrays.
            prefetched = false;
            if (k > 0) {
                const DeltaRef dn = p.d[k - 1];
                if (tid <= nt) sm.offs[ph ^ 1][tid] = dn.offsets[t_lo + tid];
                if (tid == 0) sm.next[ph ^ 1] = ~0ull;
                const long long jn = sm.cur[k - 1] + 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (jn + q * kStride < dn.count) {
                        ix[q] = __ldg(dn.indices + jn + q * kStride);
                        vx[q] = __ldg(dn.values + jn + q * kStride);
                        if (lane == 0 && jn + q * kStride > 0) px[q] = __ldg(dn.indices + jn + q * kStride - 1);
                    }
                }
                prefetched = true;
            }
            __syncthreads();  // every entry of this delta stored before the next (earlier) one
            if (tid == 0) {
                const unsigned long long nx = sm.next[ph];
                const long long end = j0 + n;
                sm.cur[k] = (nx < static_cast<unsigned long long>(end)) ? static_cast<long long>(nx) : end;
            }
        }
    }
}

}  // namespace

size_t chain_smem_bytes() { return sizeof(ChainSmem); }

cudaError_t chain_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(ChainSmem)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(chain_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(ScatSmem)));
}

cudaError_t scatter_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_scatter_kernel,
                                                         kScatThreads, sizeof(ScatSmem));
}

cudaError_t chain_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_kernel, kChainThreads,
                                                         sizeof(ChainSmem));
}

cudaError_t launch_delta_flag_clear(const WsView &ws, cudaStream_t s) {
    delta_flag_clear_kernel<<<1, 1, 0, s>>>(ws);
    return launched();
}

cudaError_t launch_delta_check(const WsView &ws, const DeltaRef *deltas, int K, cudaStream_t s) {
    cudaError_t e = launch_delta_flag_clear(ws, s);
    if (e != cudaSuccess) return e;
    CheckParams p;
    p.ws = ws;
    p.K = K;
    for (int k = 0; k < K; ++k) p.d[k] = deltas[k];
    delta_check_kernel<<<K, 256, 0, s>>>(p);
    return launched();
}

cudaError_t launch_apply(const WsView &ws, uint16_t *const *snap_ptrs, const DeltaRef &d,
                         cudaStream_t s) {
    cudaError_t e = launch_delta_check(ws, &d, 1, s);
    if (e != cudaSuccess) return e;
    if (d.count <= 0) return cudaSuccess;
    ApplyParams p;
    p.ws = ws;
    p.snap_ptrs = snap_ptrs;
    p.d = d;
    const long long blocks = (d.count + kApplyEntries - 1) / kApplyEntries;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    apply_kernel<<<static_cast<unsigned int>(blocks), kApplyThreads, 0, s>>>(p);
    return launched();
}

cudaError_t launch_apply_chain(const WsView &ws, uint16_t *const *snap_ptrs,
                               const DeltaRef *deltas, int K, long long total_entries,
                               long long total_elems, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = launch_delta_check(ws, deltas, K, s);
    if (e != cudaSuccess) return e;

    ChainParams p;
    p.ws = ws;
    p.snap_ptrs = snap_ptrs;
    p.K = K;
    for (int k = 0; k < K; ++k) p.d[k] = deltas[k];
    // Entries read per delta per round: the mean per full unit with margin,
    // a multiple of 32 (one warp's slots always belong to one delta) and
    // K * L <= kChainMaxSlots (K <= 64 keeps L >= 64).
    const double per_unit = total_elems > 0
                                ? double(total_entries) / K * kChainUnitElems / double(total_elems)
                                : 0.0;
    long long L = static_cast<long long>(per_unit * 1.25) + 32;
    L = (L + 31) & ~31LL;
    const long long cap = (kChainMaxSlots / K) & ~31LL;
    if (L > cap) L = cap;
    p.block_len = static_cast<int>(L);

    long long grid = static_cast<long long>(di.sm_count) * di.chain_ctas_per_sm;
    if (grid > ws.num_tiles) grid = ws.num_tiles;
    if (grid < 1) grid = 1;
    p.tiles_per_cta = (ws.num_tiles + grid - 1) / grid;
    grid = (ws.num_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
    chain_kernel<<<static_cast<unsigned int>(grid), kChainThreads, sizeof(ChainSmem), s>>>(p);
    return launched();
}

cudaError_t launch_apply_chain_scatter(const WsView &ws, uint16_t *const *snap_ptrs,
                                       const DeltaRef *deltas, int K, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = launch_delta_check(ws, deltas, K, s);
    if (e != cudaSuccess) return e;
    ScatParams p;
    p.ws = ws;
    p.snap_ptrs = snap_ptrs;
    p.K = K;
    for (int k = 0; k < K; ++k) p.d[k] = deltas[k];
    long long grid = static_cast<long long>(di.sm_count) * di.scatter_ctas_per_sm;
    const long long windows = (ws.num_tiles + kWinTiles - 1) / kWinTiles;
    if (grid > windows) grid = windows;
    if (grid < 1) grid = 1;
    // whole windows per CTA, so that only the last window of the plan is short
    const long long win_per_cta = (windows + grid - 1) / grid;
    p.tiles_per_cta = win_per_cta * kWinTiles;
    grid = (ws.num_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
    chain_scatter_kernel<<<static_cast<unsigned int>(grid), kScatThreads, sizeof(ScatSmem), s>>>(p);
    return launched();
}

}  // namespace dws
