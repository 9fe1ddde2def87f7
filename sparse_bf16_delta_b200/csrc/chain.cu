// chain.cu -- replay of a chain of deltas onto an anchor snapshot, in place
// ("Delta Weight Sync in TRL" §4.1: an anchor every N syncs, sparse deltas in
// between; a new replica takes the latest anchor and replays the deltas after
// it, the later delta winning where two touch the same element).
//
// Three kernels per pass over the snapshot:
//
//   chain_index_kernel  reads every entry of every delta once (coalesced
//     16-byte loads), checks it (index inside its tensor, strictly above the
//     entry before it in its tensor's segment) and writes the chain's tile
//     index: for tile g and delta k, the first entry of k at or past the start
//     of g, mod 2^32.  A failed check sets the workspace's delta flag, and the
//     replay kernels then write nothing: a chain with a bad entry anywhere is
//     not applied at all.
//
//   chain_merge_kernel  (DWS_CHAIN_TILE_MERGE) one persistent CTA per SM over
//     a contiguous range of tiles.  A producer warp fills a 4-stage ring:
//     per tile, one bulk copy of the snapshot tile and, per delta, bulk copies
//     of exactly that tile's entries (the tile index gives their range), so
//     the loads of the next tiles are in flight while 8 consumer warps merge
//     the current one: every entry of every delta raises its element's tag
//     to (k + 1) << 16 | value with atomicMax (the latest delta wins whatever
//     the thread order), then one pass moves the tagged values into the
//     tile.  The producer writes the merged tile back with one bulk store as
//     soon as it is done.  A tile no delta touches is neither read nor
//     written.
//
//   chain_scatter_kernel  (DWS_CHAIN_SCATTER) per window of 32 tiles the
//     deltas are replayed from the last to the first, an element being
//     stored only if its written-bit in shared memory is clear, so every
//     element is written once, by the latest delta that names it; untouched
//     32-byte sectors are not moved at all.  The tile index gives each
//     window's stretch of every delta.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s

// ---------------------------------------------------------------------------
// Tile index and validation
// ---------------------------------------------------------------------------
constexpr int kIdxThreads = 256;
constexpr int kIdxPerThread = 16;
constexpr int kIdxChunk = kIdxThreads * kIdxPerThread;  // entries per block step

struct IndexParams {
    WsView ws;
    DeltaRef d[DWS_MAX_CHAIN];
    int K;
    int write;                 // write the tile index (else only check)
    uint32_t *index;           // [(ntiles + 1) * kChainGroup]
};

// index rows (lo, hi] of column `col` get `v`; the warp's lanes with long
// runs fill them together, the others alone.  Every lane of the warp calls
// it (warp-wide primitives); rows outside [0, nrows] are never written.
__device__ __forceinline__ void fill_rows(uint32_t *index, int col, long long lo, long long hi,
                                          uint32_t v, int lane, long long nrows) {
    if (lo < -1) lo = -1;
    if (hi > nrows) hi = nrows;
    const bool big = hi - lo > 32;
    unsigned int m = __ballot_sync(0xffffffffu, big);
    if (!big) {
        for (long long g = lo + 1; g <= hi; ++g) index[g * kChainGroup + col] = v;
    }
    while (m != 0u) {
        const int l = __ffs(m) - 1;
        m &= m - 1;
        const long long a = __shfl_sync(0xffffffffu, lo, l);
        const long long b = __shfl_sync(0xffffffffu, hi, l);
        const uint32_t w = __shfl_sync(0xffffffffu, v, l);
        for (long long g = a + 1 + lane; g <= b; g += 32) index[g * kChainGroup + col] = w;
    }
}

// Tile of entry j (index i, tensor t), or -2 if i is outside the tensor.
__device__ __forceinline__ long long entry_tile(const IndexParams &p, int t, int i) {
    return (i >= 0 && static_cast<long long>(i) < p.ws.numel[t]) ? p.ws.first_tile[t] + (i >> kTileShift) : -2;
}

// Block (x, k): entries [x * kIdxChunk, (x + 1) * kIdxChunk) of delta k,
// 16 consecutive ones per thread.  Each thread checks its run (strictly
// ascending, inside its tensor) and writes the index rows that start at its
// entries: entry j starts rows (tile of entry j-1, tile of entry j], the last
// entry also rows (its tile, ntiles] (at n).
__global__ void __launch_bounds__(kIdxThreads, 4) chain_index_kernel(IndexParams p) {
    __shared__ int s_t[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = blockIdx.y;
    const DeltaRef d = p.d[k];
    const int T = p.ws.num_tensors;
    const long long ntiles = p.ws.num_tiles;
    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;  // offsets failed: nothing else
    const long long n = d.offsets[T];
    const long long base = static_cast<long long>(blockIdx.x) * kIdxChunk;
    if (n == 0) {  // no entry: every row points at entry 0
        if (p.write && blockIdx.x == 0 && warp == 0) fill_rows(p.index, k, -1, ntiles, 0u, lane, ntiles);
        return;
    }
    if (base >= n) return;  // uniform
    const long long last = (base + kIdxChunk < n ? base + kIdxChunk : n) - 1;
    if (warp < 2) {  // tensors of the block's first and last entries
        const int t = warp_tensor_of_entry(d.offsets, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    // this thread's entries and the one before them, in flight meanwhile
    const long long j0 = base + static_cast<long long>(tid) * kIdxPerThread;
    const bool live0 = j0 <= last;
    const int nlive = !live0 ? 0 : static_cast<int>(last - j0 + 1 < kIdxPerThread ? last - j0 + 1 : kIdxPerThread);
    int x[kIdxPerThread];
    if (nlive == kIdxPerThread && (reinterpret_cast<uintptr_t>(d.indices) & 15u) == 0) {
#pragma unroll
        for (int v = 0; v < kIdxPerThread / 4; ++v) {
            const int4 a = __ldg(reinterpret_cast<const int4 *>(d.indices + j0) + v);
            x[4 * v] = a.x; x[4 * v + 1] = a.y; x[4 * v + 2] = a.z; x[4 * v + 3] = a.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < kIdxPerThread; ++q) x[q] = (q < nlive) ? __ldg(d.indices + j0 + q) : 0;
    }
    const int prev = (live0 && j0 > 0) ? __ldg(d.indices + j0 - 1) : 0;
    __syncthreads();
    const int t0 = s_t[0], t1 = s_t[1];

    bool bad = false;
    long long bad_j = 0;
    long long glast = -2;  // tile of this thread's last entry
    // The path is chosen per warp (both call warp-wide primitives): the fast
    // one only if every lane's run qualifies.
    const bool fast_lane = live0 && nlive == kIdxPerThread &&
                           (t0 == t1 || d.offsets[t0 + 1] > j0 + kIdxPerThread - 1) && d.offsets[t0] <= j0;
    if (__all_sync(0xffffffffu, fast_lane)) {
        // Common case, 32-bit: the run lies in tensor t0.  It must ascend
        // strictly (one compare per entry); then it is in range if its ends
        // are.  The run's first entry may open t0's segment: no order check
        // then, and its predecessor (another tensor's) bounds its rows.
        const int t = t0;
        const int nm = static_cast<int>(p.ws.numel[t]);
        const long long ft = p.ws.first_tile[t];
        const bool opens = d.offsets[t] == j0;
        bool viol = !opens && !(prev < x[0]);
#pragma unroll
        for (int q = 1; q < kIdxPerThread; ++q) viol |= !(x[q - 1] < x[q]);
        const bool ok = !viol && x[0] >= 0 && x[kIdxPerThread - 1] < nm;
        if (!ok) {
            // rare: the first offending entry (unrolled: x stays in registers)
            unsigned int badm = 0;
#pragma unroll
            for (int q = 0; q < kIdxPerThread; ++q) {
                const int pv = q == 0 ? prev : x[q - 1];
                const bool e_ok = x[q] >= 0 && x[q] < nm && ((q == 0 && opens) || pv < x[q]);
                badm |= e_ok ? 0u : (1u << q);
            }
            bad = true;
            bad_j = j0 + (badm ? __ffs(badm) - 1 : 0);
        }
        glast = ok ? ft + (x[kIdxPerThread - 1] >> kTileShift) : -2;
        if (p.write) {
            // the tile of the entry before the run: this tensor's, or, when
            // the run opens the segment, found by a search (once per tensor)
            long long gprev = -1;
            if (j0 > 0) {
                if (!opens) {
                    gprev = ft + (prev >> kTileShift);
                } else {
                    int lo = 0, hi = t;  // the tensor of entry j0 - 1
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (d.offsets[mid] <= j0 - 1) lo = mid;
                        else hi = mid - 1;
                    }
                    gprev = entry_tile(p, lo, prev);
                }
            }
            // Rows (tile of entry q-1, tile of entry q] start at entry q, and
            // after the delta's last entry rows (its tile, ntiles] at n.  Each
            // lane writes its own short runs of rows (one row, usually);
            // runs longer than 32 rows (sparse deltas) are written by the
            // whole warp afterwards.  Bit 16 of `bigm` is the tail.
            unsigned int bigm = 0;
            const bool tail = ok && j0 + kIdxPerThread - 1 == n - 1;
            if (ok && gprev >= -1) {
                const long long g0 = ft + (x[0] >> kTileShift);
                if (g0 > gprev) {
                    if (g0 - gprev <= 32) {
                        for (long long g = gprev + 1; g <= g0; ++g)
                            p.index[g * kChainGroup + k] = static_cast<uint32_t>(j0);
                    } else {
                        bigm |= 1u;
                    }
                }
                int tp = x[0] >> kTileShift;
#pragma unroll
                for (int q = 1; q < kIdxPerThread; ++q) {
                    const int tl = x[q] >> kTileShift;
                    if (tl != tp) {
                        if (tl - tp <= 32) {
                            for (long long g = ft + tp + 1; g <= ft + tl; ++g)
                                p.index[g * kChainGroup + k] = static_cast<uint32_t>(j0 + q);
                        } else {
                            bigm |= 1u << q;
                        }
                    }
                    tp = tl;
                }
                if (tail) {
                    if (ntiles - glast <= 32) {
                        for (long long g = glast + 1; g <= ntiles; ++g)
                            p.index[g * kChainGroup + k] = static_cast<uint32_t>(n);
                    } else {
                        bigm |= 1u << 16;
                    }
                }
            }
            while (__any_sync(0xffffffffu, bigm != 0u)) {
                // one long run per lane per round, the warp writing together
                long long lo = 0, hi = 0;
                uint32_t v = 0;
                if (bigm != 0u) {
                    const int q = __ffs(bigm) - 1;
                    bigm &= bigm - 1;
                    if (q == 16) {
                        lo = glast;
                        hi = ntiles;
                        v = static_cast<uint32_t>(n);
                    } else {
                        int xi = 0, xp = 0;
#pragma unroll
                        for (int r = 0; r < kIdxPerThread; ++r) {
                            if (r == q) xi = x[r];
                            if (r == q - 1) xp = x[r];
                        }
                        hi = ft + (xi >> kTileShift);
                        lo = (q == 0) ? gprev : ft + (xp >> kTileShift);
                        v = static_cast<uint32_t>(j0 + q);
                    }
                }
                fill_rows(p.index, k, lo, hi, v, lane, ntiles);
            }
        }
    } else {
        // General case (a run across tensors, a short run, or a block that
        // the search placed oddly): every entry's tensor is walked.
        long long g[kIdxPerThread];
        unsigned int okm = 0;  // bit q: entry q in range and ordered
        long long gprev0 = -1;  // tile of the entry before the run
        int tq = t0;
        if (live0) {
            int lo = t0, hi = t1;  // the tensor of entry j0
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (d.offsets[mid] <= j0) lo = mid;
                else hi = mid - 1;
            }
            tq = lo;
            if (j0 > 0) {
                int tp = tq;
                if (d.offsets[tq] > j0 - 1 || d.offsets[tq] == j0) {
                    int a = 0, b = tq;  // the tensor of entry j0 - 1
                    while (a < b) {
                        const int mid = (a + b + 1) >> 1;
                        if (d.offsets[mid] <= j0 - 1) a = mid;
                        else b = mid - 1;
                    }
                    tp = a;
                }
                gprev0 = entry_tile(p, tp, prev);
            }
        }
        int pv = prev;
#pragma unroll
        for (int q = 0; q < kIdxPerThread; ++q) {
            const long long j = j0 + q;
            g[q] = -2;
            if (q < nlive) {
                while (d.offsets[tq + 1] <= j) ++tq;  // empty tensors are skipped too
                const int i = x[q];
                const bool ord = j == d.offsets[tq] || pv < i;
                g[q] = entry_tile(p, tq, i);
                okm |= (g[q] >= 0 && ord) ? (1u << q) : 0u;
            }
            pv = x[q];
        }
        const unsigned int livem = (1u << nlive) - 1u;
        const unsigned int badm = livem & ~okm;
        if (badm != 0u) {
            bad = true;
            bad_j = j0 + (__ffs(badm) - 1);
        }
#pragma unroll
        for (int r = 0; r < kIdxPerThread; ++r)
            if (r == nlive - 1) glast = g[r];
        if (p.write) {
            unsigned int bnd = 0;
            long long gp = gprev0;
#pragma unroll
            for (int q = 0; q < kIdxPerThread; ++q) {
                if (((livem >> q) & 1u) && g[q] >= 0 && gp >= -1 && g[q] > gp) bnd |= 1u << q;
                if ((livem >> q) & 1u) gp = g[q];
            }
            const bool tail = nlive > 0 && j0 + nlive - 1 == n - 1 && glast >= 0;
            unsigned int any_q = __reduce_or_sync(0xffffffffu, bnd);
            while (any_q != 0u) {
                const int q = __ffs(any_q) - 1;
                any_q &= any_q - 1;
                long long lo = gprev0, gq = 0;
#pragma unroll
                for (int r = 0; r < kIdxPerThread; ++r) {
                    if (r < q && ((livem >> r) & 1u)) lo = g[r];
                    if (r == q) gq = g[r];
                }
                const bool mine = (bnd >> q) & 1u;
                fill_rows(p.index, k, mine ? lo : 0, mine ? gq : 0, static_cast<uint32_t>(j0 + q), lane, ntiles);
            }
            if (__any_sync(0xffffffffu, tail))
                fill_rows(p.index, k, tail ? glast : 0, tail ? ntiles : 0, static_cast<uint32_t>(n), lane, ntiles);
        }
    }
    if (bad) {
        atomicOr(&p.ws.hdr->delta_bad, 1u);
        record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, bad_j);
    }
}

// The first entry of delta `d` at or past the start of tile g (in tensor t),
// from the tile index: the only value in [offsets[t], offsets[t+1]] with
// these low 32 bits (a tensor has fewer than 2^31 entries).
__device__ __forceinline__ long long index_entry(const DeltaRef &d, const uint32_t *index, long long g,
                                                 int col, int t) {
    const long long lo = d.offsets[t];
    return lo + static_cast<long long>(index[g * kChainGroup + col] - static_cast<uint32_t>(lo));
}

// ---------------------------------------------------------------------------
// Tile merge
// ---------------------------------------------------------------------------
constexpr int kMergeConsumerWarps = 8;
constexpr int kMergeConsumers = 32 * kMergeConsumerWarps;
constexpr int kMergeThreads = 32 + kMergeConsumers;
constexpr int kStages = 4;
constexpr int kStageEntries = 4096;  // entries staged per stage, all deltas together

struct MergeParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    const uint32_t *index;
    long long tiles_per_cta;
    int K;
    DeltaRef d[kChainGroup];
};

// What the producer staged for one tile.
struct StageMeta {
    long long s[kChainGroup];  // first entry of the tile in delta k
    int n[kChainGroup];        // entries of the tile in delta k
    int ia[kChainGroup];       // staged indices: entries s + [ia, ib) at idx[io + ...] (ia may be < 0)
    int ib[kChainGroup];
    int io[kChainGroup];
    int va[kChainGroup];       // staged values: entries s + [va, vb) at val[vo + ...]
    int vb[kChainGroup];
    int vo[kChainGroup];
    int C[kChainGroup + 1];    // work items (32 entries of one delta): delta k's are [C[k], C[k+1])
    uint16_t *ptr;  // tile start in the snapshot
    int local_start;
    int count;   // elements of the tile
    int bulk;    // leading elements moved by bulk copies (multiple of 8)
    int touched;
};

struct MergeSmem {
    uint32_t tag[kTileElems];  // (k + 1) << 16 | value of the latest delta k per element; 0: none
    uint16_t tile[kStages][kTileElems];
    int idx[kStages][kStageEntries];
    uint16_t val[kStages][kStageEntries];
    StageMeta meta[kStages];
    unsigned long long full[kStages];  // producer -> consumers: tile staged
    unsigned long long done[kStages];  // consumers -> producer: tile merged
    int grp[kStages];                  // producer: store group of the stage's tile (-1: none)
    long long cursor[kChainGroup];
    int abort;
};

// Producer warp's view of the tensor that holds the current tile.
struct TensorCursor {
    int t;              // tensor
    long long first;    // its first tile
    long long next;     // first tile of the next tensor
    long long numel;
    uint16_t *ptr;
};

__device__ __forceinline__ void tensor_at(const MergeParams &p, int t, TensorCursor &c) {
    c.t = t;
    c.first = p.ws.first_tile[t];
    c.next = p.ws.first_tile[t + 1];
    c.numel = p.ws.numel[t];
    c.ptr = p.snap_ptrs[t];
}

// Producer warp: describe tile i and start its copies into stage st.  Lane k
// (< K) owns delta k: its entries of the tile are [cursor, cursor + n) with
// n the difference of two index rows (mod 2^32; a tile holds fewer).
__device__ void merge_stage(const MergeParams &p, MergeSmem &sm, long long i, int st,
                            const TensorCursor &tc, uint32_t row_next, long long &cursor,
                            unsigned long long policy) {
    const int lane = threadIdx.x & 31;
    StageMeta &m = sm.meta[st];
    const long long ls = (i - tc.first) << kTileShift;
    const long long rest = tc.numel - ls;
    const int count = static_cast<int>(rest < kTileElems ? (rest > 0 ? rest : 0) : kTileElems);
    const bool mine = lane < p.K;
    int n = 0;
    long long s = 0;
    if (mine) {
        s = cursor;
        const uint32_t row_here = static_cast<uint32_t>(s);  // the row of tile i, as cursor's low bits
        n = static_cast<int>(row_next - row_here);
        cursor = s + n;
    }
    int total = n;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    const uintptr_t ua = reinterpret_cast<uintptr_t>(tc.ptr);
    bool touched = total > 0 && count > 0;
    if (touched && (tc.ptr == nullptr || (ua & 1u))) {
        if (lane == 0) record_error(p.ws.hdr, DWS_ERR_INVALID, tc.t);
        touched = false;
    }
    const int bulk = (touched && (ua & 15u) == 0) ? (count & ~7) : 0;
    // Entries: each delta's range widened to 16-byte boundaries (so that
    // no entry of the tile has to come from global memory), kept inside the
    // delta's arrays: only at the arrays' unaligned ends do a few entries
    // stay outside it.  A prefix sum over the lanes places the ranges while
    // there is room.
    int ci = 0, cv = 0;
    long long ia = 0, va = 0;  // absolute first staged entry
    if (mine && touched && n > 0) {
        const DeltaRef &dk = p.d[lane];
        const uintptr_t lo_i = (reinterpret_cast<uintptr_t>(dk.indices) + 15) & ~uintptr_t(15);
        const uintptr_t hi_i = reinterpret_cast<uintptr_t>(dk.indices + dk.count) & ~uintptr_t(15);
        uintptr_t a = reinterpret_cast<uintptr_t>(dk.indices + s) & ~uintptr_t(15);
        uintptr_t b = (reinterpret_cast<uintptr_t>(dk.indices + s + n) + 15) & ~uintptr_t(15);
        if (a < lo_i) a = lo_i;
        if (b > hi_i) b = hi_i;
        if (b > a && ((a - reinterpret_cast<uintptr_t>(dk.indices)) & 3u) == 0) {
            ci = static_cast<int>((b - a) >> 2);
            ia = static_cast<long long>((a - reinterpret_cast<uintptr_t>(dk.indices)) >> 2);
        }
        const uintptr_t lo_v = (reinterpret_cast<uintptr_t>(dk.values) + 15) & ~uintptr_t(15);
        const uintptr_t hi_v = reinterpret_cast<uintptr_t>(dk.values + dk.count) & ~uintptr_t(15);
        uintptr_t c = reinterpret_cast<uintptr_t>(dk.values + s) & ~uintptr_t(15);
        uintptr_t d = (reinterpret_cast<uintptr_t>(dk.values + s + n) + 15) & ~uintptr_t(15);
        if (c < lo_v) c = lo_v;
        if (d > hi_v) d = hi_v;
        if (d > c && ((c - reinterpret_cast<uintptr_t>(dk.values)) & 1u) == 0) {
            cv = static_cast<int>((d - c) >> 1);
            va = static_cast<long long>((c - reinterpret_cast<uintptr_t>(dk.values)) >> 1);
        }
    }
    int oi = ci, ov = cv;  // inclusive prefix over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, oi, o);
        const int y = __shfl_up_sync(0xffffffffu, ov, o);
        if (lane >= o) {
            oi += x;
            ov += y;
        }
    }
    oi -= ci;  // exclusive
    ov -= cv;
    if (oi + ci > kStageEntries) ci = oi < kStageEntries ? ((kStageEntries - oi) & ~3) : 0;
    if (ov + cv > kStageEntries) cv = ov < kStageEntries ? ((kStageEntries - ov) & ~7) : 0;
    int fn = (n + 31) >> 5;  // inclusive prefix of the work items over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, fn, o);
        if (lane >= o) fn += x;
    }
    if (lane < p.K) m.C[lane + 1] = fn;
    if (lane == 0) m.C[0] = 0;
    if (mine) {
        m.s[lane] = s;
        m.n[lane] = n;
        // staged ranges relative to s (may start before it)
        m.ia[lane] = static_cast<int>(ia - s);
        m.ib[lane] = static_cast<int>(ia - s) + ci;
        m.io[lane] = oi;
        m.va[lane] = static_cast<int>(va - s);
        m.vb[lane] = static_cast<int>(va - s) + cv;
        m.vo[lane] = ov;
    }
    uint32_t bytes = static_cast<uint32_t>(ci) * 4u + static_cast<uint32_t>(cv) * 2u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
    if (lane == 0) {
        m.ptr = touched ? tc.ptr + ls : nullptr;
        m.local_start = static_cast<int>(ls);
        m.count = count;
        m.bulk = bulk;
        m.touched = touched ? 1 : 0;
    }
    __syncwarp();
    if (lane == 0) {
        bytes += static_cast<uint32_t>(bulk) * 2u;
        mbar_arrive_expect_tx(&sm.full[st], bytes);  // releases the description above
        if (bulk > 0)
            bulk_load(sm.tile[st], tc.ptr + ls, static_cast<uint32_t>(bulk) * 2u, &sm.full[st], policy);
    }
    __syncwarp();
    if (ci > 0)
        bulk_load(&sm.idx[st][oi], p.d[lane].indices + ia, static_cast<uint32_t>(ci) * 4u,
                  &sm.full[st], policy);
    if (cv > 0)
        bulk_load(&sm.val[st][ov], p.d[lane].values + va, static_cast<uint32_t>(cv) * 2u,
                  &sm.full[st], policy);
}

__global__ void __launch_bounds__(kMergeThreads, 1) chain_merge_kernel(MergeParams p) {
    extern __shared__ __align__(128) unsigned char merge_smem_raw[];
    MergeSmem &sm = *reinterpret_cast<MergeSmem *>(merge_smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (!ws_matches(p.ws)) return;
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;
    const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_cta;
    long long te = tb + p.tiles_per_cta;
    if (te > p.ws.num_tiles) te = p.ws.num_tiles;
    if (tb >= te) return;
    const long long ntl = te - tb;

    if (tid == 0) {
        sm.abort = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.done[s], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---- producer warp ---------------------------------------------------
        // Stages tile li once tile li - kStages is merged and its store has
        // read the stage; stores are issued as soon as a tile is merged.
        const unsigned long long policy = l2_evict_first_policy();
        TensorCursor tc;
        tensor_at(p, p.ws.tile_tensor[tb], tc);
        long long cursor = 0;  // lane k: delta k's first entry of the next tile to stage
        uint32_t rq0 = 0, rq1 = 0, rq2 = 0, rq3 = 0;  // index rows of tiles i+1 .. i+4
        const long long nrows = p.ws.num_tiles;      // last row
        if (lane < p.K) {
            cursor = index_entry(p.d[lane], p.index, tb, lane, tc.t);
            rq0 = p.index[(tb + 1) * kChainGroup + lane];
            if (tb + 2 <= nrows) rq1 = p.index[(tb + 2) * kChainGroup + lane];
            if (tb + 3 <= nrows) rq2 = p.index[(tb + 3) * kChainGroup + lane];
            if (tb + 4 <= nrows) rq3 = p.index[(tb + 4) * kChainGroup + lane];
        }
        long long taken = 0;  // tiles whose completion the producer has taken
        int committed = 0;    // store groups committed
        // take tile c's completion: write it back
        auto take = [&](long long c) {
            const int cs = static_cast<int>(c % kStages);
            const StageMeta &m = sm.meta[cs];
            if (m.touched && m.bulk > 0) {
                bulk_store(m.ptr, sm.tile[cs], static_cast<uint32_t>(m.bulk) * 2u);
                bulk_commit();
                sm.grp[cs] = committed++;
            } else {
                sm.grp[cs] = -1;
            }
        };
        bool ok = true;
        for (long long li = 0; li < ntl; ++li) {
            const long long i = tb + li;
            const int st = static_cast<int>(li % kStages);
            while (i >= tc.next) tensor_at(p, tc.t + 1, tc);  // uniform
            if (lane == 0) {
                while (taken < li && mbar_try_wait(&sm.done[taken % kStages],
                                                   static_cast<uint32_t>((taken / kStages) & 1)))
                    take(taken++);
                while (ok && taken <= li - kStages) {
                    ok = mbar_wait_sleepy(&sm.done[taken % kStages], static_cast<uint32_t>((taken / kStages) & 1),
                                          kWaitLimitNs);
                    if (ok) take(taken++);
                }
                if (ok && li >= kStages && sm.grp[st] >= 0) bulk_wait_read_n(committed - 1 - sm.grp[st]);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            __syncwarp();
            merge_stage(p, sm, i, st, tc, rq0, cursor, policy);
            rq0 = rq1;
            rq1 = rq2;
            rq2 = rq3;
            rq3 = (lane < p.K && i + 5 <= nrows) ? p.index[(i + 5) * kChainGroup + lane] : 0u;
        }
        if (lane == 0) {
            // write back the last tiles
            while (ok && taken < ntl) {
                ok = mbar_wait_sleepy(&sm.done[taken % kStages], static_cast<uint32_t>((taken / kStages) & 1),
                                      kWaitLimitNs);
                if (ok) take(taken++);
            }
            if (!ok) {
                atomicExch(&sm.abort, 1);
                record_error(p.ws.hdr, DWS_ERR_TIMEOUT, tb);
            }
            bulk_wait_all();
        }
        return;
    }

    // ---- consumers (8 warps) ------------------------------------------------
    // Per tile: the entries of all deltas as one list; each entry raises its
    // element's tag to (k + 1) << 16 | value with atomicMax, so the latest
    // delta wins whatever the order the threads run in; then one pass moves
    // the tagged values into the tile (or straight to global memory past the
    // bulk-copied part) and clears the tags.
    const int ct = tid - 32;  // 0 .. kMergeConsumers - 1
    for (int e = ct; e < kTileElems; e += kMergeConsumers) sm.tag[e] = 0u;
    named_bar(1, kMergeConsumers);
    for (long long li = 0; li < ntl; ++li) {
        const int st = static_cast<int>(li % kStages);
        const bool got = mbar_wait_sleepy(&sm.full[st], static_cast<uint32_t>((li / kStages) & 1), kWaitLimitNs);
        if (!named_bar_and(1, kMergeConsumers, got && ld_acquire_cta(&sm.abort) == 0)) {
            if (ct == 0) record_error(p.ws.hdr, DWS_ERR_TIMEOUT, tb + li);
            return;  // the producer's own waits are bounded too
        }
        const StageMeta &m = sm.meta[st];
        if (m.touched) {
            const int ls = m.local_start;
            const int count = m.count;
            const int items = m.C[p.K];
            const int cw = ct >> 5;
            int k = -1, c_lo = 0, c_hi = 0, n = 0, ia = 0, ib = 0, io = 0, va = 0, vb = 0, vo = 0;
            bool staged = false;
            const int *gi = nullptr;
            const uint16_t *gv = nullptr;
            for (int it = cw; it < items; it += kMergeConsumerWarps) {
                while (it >= c_hi) {  // uniform per warp: items only move forward
                    ++k;
                    c_lo = m.C[k];
                    c_hi = m.C[k + 1];
                    n = m.n[k];
                    ia = m.ia[k]; ib = m.ib[k]; io = m.io[k];
                    va = m.va[k]; vb = m.vb[k]; vo = m.vo[k];
                    staged = ia <= 0 && ib >= n && va <= 0 && vb >= n;
                    gi = p.d[k].indices + m.s[k];
                    gv = p.d[k].values + m.s[k];
                }
                const int el = ((it - c_lo) << 5) + lane;
                if (el >= n) continue;
                int ix;
                uint32_t vx;
                if (staged) {
                    ix = sm.idx[st][io + el - ia];
                    vx = sm.val[st][vo + el - va];
                } else {
                    // outside the staged range: from global memory, inside the
                    // delta's arrays whatever the index says
                    const bool in_arr = m.s[k] + el >= 0 && m.s[k] + el < p.d[k].count;
                    ix = (el >= ia && el < ib) ? sm.idx[st][io + el - ia] : (in_arr ? __ldg(gi + el) : -1);
                    vx = (el >= va && el < vb) ? sm.val[st][vo + el - va] : (in_arr ? __ldg(gv + el) : 0u);
                }
                const int pos = ix - ls;  // in [0, count): the index pass's ranges
                if (static_cast<unsigned>(pos) < static_cast<unsigned>(count))
                    atomicMax(&sm.tag[pos], (static_cast<uint32_t>(k + 1) << 16) | vx);
                else
                    record_error(p.ws.hdr, DWS_ERR_WORKSPACE, m.s[k] + el);  // never expected
            }
            named_bar(1, kMergeConsumers);
            const int bulk = m.bulk;
            uint16_t *tile = sm.tile[st];
#pragma unroll
            for (int r = 0; r < kTileElems / (4 * kMergeConsumers); ++r) {
                const int e0 = 4 * ct + r * 4 * kMergeConsumers;
                if (e0 >= count) break;
                const uint4 tg = *reinterpret_cast<const uint4 *>(&sm.tag[e0]);
                if ((tg.x | tg.y | tg.z | tg.w) == 0u) continue;
                *reinterpret_cast<uint4 *>(&sm.tag[e0]) = make_uint4(0u, 0u, 0u, 0u);
                const uint32_t t4[4] = {tg.x, tg.y, tg.z, tg.w};
                if (e0 + 4 <= bulk) {
                    uint2 w = *reinterpret_cast<const uint2 *>(&tile[e0]);
                    uint32_t lo = w.x, hi = w.y;
                    if (t4[0]) lo = (lo & 0xffff0000u) | (t4[0] & 0xffffu);
                    if (t4[1]) lo = (lo & 0x0000ffffu) | (t4[1] << 16);
                    if (t4[2]) hi = (hi & 0xffff0000u) | (t4[2] & 0xffffu);
                    if (t4[3]) hi = (hi & 0x0000ffffu) | (t4[3] << 16);
                    *reinterpret_cast<uint2 *>(&tile[e0]) = make_uint2(lo, hi);
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (!t4[q] || e0 + q >= count) continue;
                        if (e0 + q < bulk) tile[e0 + q] = static_cast<uint16_t>(t4[q] & 0xffffu);
                        else m.ptr[e0 + q] = static_cast<uint16_t>(t4[q] & 0xffffu);
                    }
                }
            }
            if (bulk > 0) fence_proxy_async_smem();  // the bulk store reads the tile
            named_bar(1, kMergeConsumers);
        }
        if (ct == 0) mbar_arrive(&sm.done[st]);
    }
    if (ct == 0) {
    }
}

// ---------------------------------------------------------------------------
// Reverse-order scatter over windows, with a written-bitmap
// ---------------------------------------------------------------------------
constexpr int kScatThreads = 1024;
constexpr int kScatWarps = kScatThreads / 32;
constexpr int kWinTiles = 32;
constexpr int kWinElems = kWinTiles * kTileElems;
constexpr int kScatDepth = 4;

struct ScatParams {
    WsView ws;
    uint16_t *const *snap_ptrs;
    const uint32_t *index;
    long long tiles_per_cta;
    int K;
    DeltaRef d[kChainGroup];
};

struct ScatSmem {
    uint32_t written[kWinElems / 32];
    long long cur[kChainGroup];      // per delta: first entry of the current window
    long long len[kChainGroup];      // per delta: entries of the current window
    long long base[kWinTiles];       // per window tensor: (first_tile - window start) * tile
    long long numel[kWinTiles];
    uint16_t *ptr[kWinTiles];
    long long offs[2][kWinTiles + 1];  // a delta's offsets of the window tensors (by parity)
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

    if (tid < p.K) sm.cur[tid] = index_entry(p.d[tid], p.index, tb, tid, p.ws.tile_tensor[tb]);

    for (long long a = tb; a < te; a += kWinTiles) {
        const long long b = (a + kWinTiles < te) ? a + kWinTiles : te;
        const int win_words = static_cast<int>(b - a) * (kTileElems / 32);
        const int t_lo = p.ws.tile_tensor[a];
        const int nt = p.ws.tile_tensor[b - 1] - t_lo + 1;  // <= b - a: every tensor owns a tile
        if (t_lo < 0 || nt < 1 || nt > kWinTiles || t_lo + nt > p.ws.num_tensors) {
            if (tid == 0) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, a);
            return;  // uniform: every thread read the same table entries
        }
        __syncthreads();  // the previous window is complete
        if (p.K > 1)
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
        if (tid < p.K) {
            const int tn = b < p.ws.num_tiles ? p.ws.tile_tensor[b] : p.ws.num_tensors - 1;
            sm.len[tid] = index_entry(p.d[tid], p.index, b, tid, tn) - sm.cur[tid];
        }
        constexpr long long kStride = 32LL * kScatWarps;
        if (tid <= nt) sm.offs[(p.K - 1) & 1][tid] = p.d[p.K - 1].offsets[t_lo + tid];
        __syncthreads();

        int ix[kScatDepth];
        uint16_t vx[kScatDepth];
        bool prefetched = false;  // the phase's first chunks already requested (uniform)
        for (int k = p.K - 1; k >= 0; --k) {
            const DeltaRef d = p.d[k];
            const int ph = k & 1;
            const long long *offs = sm.offs[ph];
            // the window's stretch of delta k, kept inside its arrays
            const long long j0 = sm.cur[k] < 0 ? 0 : (sm.cur[k] > d.count ? d.count : sm.cur[k]);
            const long long nl = sm.len[k] < 0 ? 0 : (j0 + sm.len[k] > d.count ? d.count - j0 : sm.len[k]);
            const int n = static_cast<int>(nl < kWinElems ? nl : kWinElems);  // one window of one delta
            const int *pi = d.indices + j0;
            const uint16_t *pv = d.values + j0;
            int r = 32 * warp + lane;  // this lane's entry of the current chunk
            if (!prefetched) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (r + q * kStride < n) {
                        ix[q] = __ldg(pi + r + q * kStride);
                        vx[q] = __ldg(pv + r + q * kStride);
                    }
                }
            }
            // The warp's current tensor (its chunks only move forward) and
            // that tensor's constants: segment end relative to j0, window
            // offset, size, pointer.
            int tw = 0;
            while (tw + 1 < nt && offs[tw + 1] <= j0 + r - lane) ++tw;
            long long seg_hi = offs[tw + 1] - j0;
            int off_c = static_cast<int>(-sm.base[tw]);
            uint16_t *ptr_c = sm.ptr[tw];
            for (bool more = r - lane < n; more;) {
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    const int cs = r - lane;
                    if (cs >= n) {  // the whole chunk is past the stretch (uniform)
                        more = false;
                        break;
                    }
                    const int idx = ix[q];
                    const uint16_t val = vx[q];
                    if (r + kScatDepth * kStride < n) {
                        ix[q] = __ldg(pi + r + kScatDepth * kStride);
                        vx[q] = __ldg(pv + r + kScatDepth * kStride);
                    }
                    const bool valid = r < n;
                    if (cs >= seg_hi) {  // uniform: move to the chunk's first tensor
                        while (tw + 1 < nt && offs[tw + 1] <= j0 + cs) ++tw;
                        seg_hi = offs[tw + 1] - j0;
                        off_c = static_cast<int>(-sm.base[tw]);
                        ptr_c = sm.ptr[tw];
                    }
                    const int cl = (cs + 31 < n) ? cs + 31 : n - 1;
                    uint32_t rel = 0;  // element within the window
                    uint16_t *dst = ptr_c;
                    if (cl < seg_hi) {
                        // The chunk lies in one tensor (checked entries:
                        // 0 <= idx - off_c < window length).
                        rel = static_cast<uint32_t>(idx - off_c);
                    } else if (valid) {
                        const long long j = j0 + r;
                        int tl = tw;
                        while (tl + 1 < nt && offs[tl + 1] <= j) ++tl;
                        rel = static_cast<uint32_t>(sm.base[tl] + idx);
                        dst = sm.ptr[tl];
                    }
                    if (valid && rel >= static_cast<uint32_t>(kWinElems)) {  // never expected
                        record_error(p.ws.hdr, DWS_ERR_WORKSPACE, j0 + r);
                        rel = 0;
                        dst = nullptr;
                    }
                    bool store = valid;
                    if (p.K > 1) {  // uniform: a single delta needs no written-bits
                        const uint32_t word = rel >> 5;
                        const uint32_t bit = 1u << (rel & 31u);
                        if (valid) store = (sm.written[word] & bit) == 0u;
                        // Mark this delta's elements: one OR per lane, or two
                        // for a run of 32 consecutive elements (a clustered
                        // change), where per-lane ORs would all hit one word.
                        const uint32_t r0 = __shfl_sync(0xffffffffu, rel, 0);
                        const uint32_t r31 = __shfl_sync(0xffffffffu, rel, 31);
                        bool marked = false;
                        if (r31 - r0 == 31u && cs + 31 < n) {  // uniform; entries ascend
                            if (lane == 0) atomicOr(&sm.written[r0 >> 5], ~0u << (r0 & 31u));
                            if (lane == 31 && (r31 & 31u) != 31u)
                                atomicOr(&sm.written[r31 >> 5], (2u << (r31 & 31u)) - 1u);
                            marked = true;
                        }
                        if (!marked && valid) atomicOr(&sm.written[word], bit);
                    }
                    if (store && dst != nullptr) dst[idx] = val;
                    r += kStride;
                }
            }
            // This warp is done with delta k.  While the others finish,
            // request the next (earlier) delta's offsets and first chunks.
            prefetched = false;
            if (k > 0) {
                const DeltaRef dn = p.d[k - 1];
                if (tid <= nt) sm.offs[ph ^ 1][tid] = dn.offsets[t_lo + tid];
                const long long jn = sm.cur[k - 1] < 0 ? 0 : (sm.cur[k - 1] > dn.count ? dn.count : sm.cur[k - 1]);
                const long long nn0 = sm.len[k - 1] < 0 ? 0 : (jn + sm.len[k - 1] > dn.count ? dn.count - jn : sm.len[k - 1]);
                const long long nn = nn0 < kWinElems ? nn0 : kWinElems;
                const int rn = 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < kScatDepth; ++q) {
                    if (rn + q * kStride < nn) {
                        ix[q] = __ldg(dn.indices + jn + rn + q * kStride);
                        vx[q] = __ldg(dn.values + jn + rn + q * kStride);
                    }
                }
                prefetched = true;
            }
            __syncthreads();  // every entry of this delta stored before the next (earlier) one
        }
        if (tid < p.K) sm.cur[tid] += sm.len[tid];
    }
}

}  // namespace

cudaError_t chain_set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(chain_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(MergeSmem)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(chain_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(ScatSmem)));
}

cudaError_t chain_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_merge_kernel, kMergeThreads,
                                                         sizeof(MergeSmem));
}

cudaError_t index_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_index_kernel, kIdxThreads, 0);
}

cudaError_t scatter_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, chain_scatter_kernel,
                                                         kScatThreads, sizeof(ScatSmem));
}

cudaError_t launch_apply_chain(const WsView &ws, uint16_t *const *snap_ptrs, const DeltaRef *deltas,
                               int K, bool merge, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = launch_delta_check(ws, deltas, K, s);  // offsets of every delta
    if (e != cudaSuccess) return e;
    uint32_t *index = reinterpret_cast<uint32_t *>(ws.tile_status);

    // Index-pass grid: one block per kIdxChunk entries of every delta.
    auto index_grid = [&](const DeltaRef *ds, int nk, IndexParams &) -> long long {
        long long max_n = 1;
        for (int k = 0; k < nk; ++k) max_n = ds[k].count > max_n ? ds[k].count : max_n;
        return (max_n + kIdxChunk - 1) / kIdxChunk;
    };
    IndexParams ip;
    ip.ws = ws;
    ip.index = index;
    if (K > kChainGroup) {  // every delta checked before the first pass writes
        ip.K = K;
        ip.write = 0;
        for (int k = 0; k < K; ++k) ip.d[k] = deltas[k];
        const long long bx = index_grid(deltas, K, ip);
        if (bx > 0x7fffffffLL) return cudaErrorInvalidValue;
        chain_index_kernel<<<dim3(static_cast<unsigned int>(bx), K), kIdxThreads, 0, s>>>(ip);
        e = launched();
        if (e != cudaSuccess) return e;
    }
    for (int k0 = 0; k0 < K; k0 += kChainGroup) {
        const int kg = (K - k0 < kChainGroup) ? K - k0 : kChainGroup;
        ip.K = kg;
        ip.write = 1;
        for (int k = 0; k < kg; ++k) ip.d[k] = deltas[k0 + k];
        const long long gx = index_grid(deltas + k0, kg, ip);
        if (gx > 0x7fffffffLL) return cudaErrorInvalidValue;
        chain_index_kernel<<<dim3(static_cast<unsigned int>(gx), kg), kIdxThreads, 0, s>>>(ip);
        e = launched();
        if (e != cudaSuccess) return e;
        if (merge) {
            MergeParams mp;
            mp.ws = ws;
            mp.snap_ptrs = snap_ptrs;
            mp.index = index;
            mp.K = kg;
            for (int k = 0; k < kg; ++k) mp.d[k] = deltas[k0 + k];
            long long grid = static_cast<long long>(di.sm_count) * di.chain_ctas_per_sm;
            if (grid > ws.num_tiles) grid = ws.num_tiles;
            if (grid < 1) grid = 1;
            mp.tiles_per_cta = (ws.num_tiles + grid - 1) / grid;
            grid = (ws.num_tiles + mp.tiles_per_cta - 1) / mp.tiles_per_cta;
            chain_merge_kernel<<<static_cast<unsigned int>(grid), kMergeThreads, sizeof(MergeSmem), s>>>(mp);
        } else {
            ScatParams sp;
            sp.ws = ws;
            sp.snap_ptrs = snap_ptrs;
            sp.index = index;
            sp.K = kg;
            for (int k = 0; k < kg; ++k) sp.d[k] = deltas[k0 + k];
            long long grid = static_cast<long long>(di.sm_count) * di.scatter_ctas_per_sm;
            const long long windows = (ws.num_tiles + kWinTiles - 1) / kWinTiles;
            if (grid > windows) grid = windows;
            if (grid < 1) grid = 1;
            // whole windows per CTA, so that only the last window of the plan is short
            const long long win_per_cta = (windows + grid - 1) / grid;
            sp.tiles_per_cta = win_per_cta * kWinTiles;
            grid = (ws.num_tiles + sp.tiles_per_cta - 1) / sp.tiles_per_cta;
            chain_scatter_kernel<<<static_cast<unsigned int>(grid), kScatThreads, sizeof(ScatSmem), s>>>(sp);
        }
        e = launched();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace dws
