// encode.cu -- fused change detection, scan and compaction (one launch).
//
// What it computes ([verl] review, key source snippets, sparse_gather.py,
// shard_delta_indices; "Delta Weight Sync in TRL" §4.1/§4.2): for every
// tensor of the plan, the ascending local indices i where the 16-bit pattern
// of new[i] differs from old[i], and new[i] at those indices, concatenated in
// plan order with a per-tensor offsets[] prefix.
//
// How (single pass over both snapshots, 4 bytes read per element):
//   * A prepare pass (one thread per tile) clears the scan state and writes a
//     32-byte descriptor per tile: pointers to the tile in both snapshots,
//     tensor, local start, element count.
//   * One persistent CTA per SM, warp-specialised.  Tiles of 8192 elements
//     are taken by atomic ticket, so a tile's predecessors are always
//     resident or finished (forward progress of the scan below).
//   * Producer (one thread): takes tickets and reads tile descriptors two
//     tiles ahead, and refills each of the kStages stages as soon as it is
//     released: two 1-D bulk async copies (cp.async.bulk, global -> own
//     shared memory, mbarrier transaction count, L2 evict-first) bring both
//     snapshots' 16 KiB of the tile.
//   * Two counting groups of 8 warps take the stage fills in turn (group g
//     the fills g, g + 2, ...), so two tiles are counted at once and one
//     group's barriers and latencies overlap the other's work.  Eight warps
//     a group (32 elements a thread) keep a stage busy for half the time
//     four did, which matters most when many elements change: each thread
//     moves its own changed entries into the ring.  Per tile:
//     detect, block scan, publish the tile's count, move the changed
//     (offset, value) pairs into the group's shared ring, queue the tile,
//     release the stage.  A stage is busy only from its refill to its
//     count, and a tile's count never waits on any look-back: a ticket held
//     while its CTA waits on a look-back makes every later tile wait on it
//     in turn (convoys), and a stage held through a look-back caps the data
//     in flight.
//   * Look-back group (3 warps): each takes queued tiles in turn, resolves
//     the tile's exclusive prefix, publishes it, writes the tile's entries
//     from the ring with consecutive lanes storing consecutive entries
//     (coalesced), and releases its ring space.
//   * detect: 16-byte shared-memory reads in a bank-conflict-free order, a
//     32-bit change mask per thread, popc; block scan of the counts.
//   * scan: decoupled look-back over the tile status words (flag + 62-bit
//     count), one word per 32-byte sector so that the words every look-back
//     reads (the newest tiles') spread over four times as many L2 lines.  A
//     look-back reads the 32 nearest predecessors in one coalesced row, the
//     next 224 only if those are all aggregates, and while waiting re-reads
//     only the words still unpublished, with a backoff of 2 to 4 us
//     (re-reading whole windows, or often, from every waiting warp floods
//     the L2 slices holding the hottest lines, and every bulk copy through
//     those slices waits).  Bounded by a wall-clock limit after which the
//     kernel records DWS_ERR_TIMEOUT and every CTA leaves.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kGroups = 2;      // counting groups; group g counts stage fills g, g + 2, ...
constexpr int kGroupWarps = 8;  // warps per counting group
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kCountWarps = kGroups * kGroupWarps;
constexpr int kElemsPerThread = kTileElems / kGroupThreads;  // 32
constexpr int kLookWarps = 3;                     // the look-back group
constexpr int kProducerWarp = kCountWarps + kLookWarps;
constexpr int kPublishThread = 64;  // of a group: publishes tile counts (its thread 0 keeps the queue)
constexpr int kThreads = 32 * (kProducerWarp + 1);
constexpr int kStages = 4;
constexpr int kRing = 8192;  // per group: pending (offset | value << 16) entries
constexpr int kQueue = 64;   // pending tiles
constexpr int kCountBar = 1;  // named barrier of group g: kCountBar + g
static_assert(kElemsPerThread == 32, "each counting thread owns 4 chunks of 8 elements");
static_assert(kStages % kGroups == 0, "a stage always serves the same group");
static_assert((kRing & (kRing - 1)) == 0 && kRing >= kTileElems, "ring holds any tile");

constexpr unsigned long long kLoadWaitLimitNs = 4000000000ull;  // 4 s

struct StageMeta {
    long long ticket;  // >= num_tiles: no more work for this stage
    TileDesc d;
};

struct Pending {
    long long ticket;
    int tensor;
    int local_start;
    int group;  // whose ring holds the entries
    int pos;    // first ring entry
    int total;  // changed elements (ring entries when compacting)
};

struct EncodeParams {
    WsView ws;
    long long *offsets;
    int *indices;
    uint16_t *values;
    long long capacity;
    long long wait_limit_ns;
    long long withhold;
    int vec_out;  // indices 16-byte and values 8-byte aligned: entries leave four at a time
    long long *indices64;          // global positions (dws_encode_global), else null
    const long long *index_base;   // per tensor: added to the local index (global positions)
    unsigned long long *hashes;    // wire checksum halves (dws_encode_checksum), else null
};

struct EncodeSmem {
    uint16_t buf[kStages][2][kTileElems];  // [stage][old | new]
    uint32_t ring[kGroups][kRing];
    unsigned long long bar[kStages];        // stage filled (transaction count)
    unsigned long long empty_bar[kStages];  // stage released by the counting group
    int fills[kStages];                     // fills issued per stage
    int producer_done;
    StageMeta meta[kStages];
    Pending q[kQueue];
    int q_ready[kQueue];  // i + 1 once queue entry i is complete (release)
    int q_done[kQueue];   // i + 1 once queue entry i is written out
    int q_final;          // number of tiles once counting has finished, else INT_MAX
    int stop;             // a look-back gave up: everyone leaves
    int alloc_pos[kGroups];  // ring position of the group's tile, -1 = leave
    int ring_free[kGroups];  // ring entries known to be free when the tile was taken
    int warp_sum[kGroups][kGroupWarps];
};

// Thread 0, in two steps: take a ticket (early, so its latency hides behind
// a tile's work), then read its descriptor and start the stage's loads.
__device__ __forceinline__ long long take_ticket(const EncodeParams &p) {
    return static_cast<long long>(atomicAdd(&p.ws.hdr->ticket, 1ull));
}

__device__ __forceinline__ TileDesc load_desc(const EncodeParams &p, long long ticket) {
    TileDesc d;
    if (ticket < p.ws.num_tiles) {
        d = p.ws.tile_desc[ticket];
    } else {
        d.old_p = nullptr;
        d.new_p = nullptr;
        d.tensor = 0;
        d.local_start = 0;
        d.count = 0;
        d.bulk = 0;
    }
    return d;
}

__device__ void issue_stage(const EncodeParams &p, EncodeSmem &sm, int s, long long ticket,
                            const TileDesc &desc) {
    StageMeta m;
    m.ticket = ticket;
    m.d = desc;
    sm.meta[s] = m;
    sm.fills[s] += 1;
    if (ticket < p.ws.num_tiles) {
        const uint32_t bulk = static_cast<uint32_t>(m.d.bulk);
        mbar_arrive_expect_tx(&sm.bar[s], bulk * 4u);  // release: meta is visible
        if (bulk > 0) {
            const unsigned long long policy = l2_evict_first_policy();
            bulk_load(sm.buf[s][0], m.d.old_p, bulk * 2u, &sm.bar[s], policy);
            bulk_load(sm.buf[s][1], m.d.new_p, bulk * 2u, &sm.bar[s], policy);
        }
    } else {
        mbar_arrive(&sm.bar[s]);  // no more work: wake the counting group
    }
}

// Decoupled look-back, run by one warp.  Row q of a window holds the 32
// predecessors at distances 32q + lane (so a row is one coalesced read of
// 256 bytes, 8 sectors), nearest row first.  The nearest row is read alone
// first; the other seven only if it holds neither a prefix nor an
// unpublished word.  The nearest word that is a prefix ends the look-back
// (the aggregates before it are summed); the nearest unpublished word
// blocks it, and while blocked only the unpublished words before the first
// prefix are read again (with backoff): an aggregate stays valid even after
// it turns into a prefix, and re-reading whole windows from every waiting
// warp floods the L2 with requests to the hottest lines.  Returns -1 if the
// bounded wait ran out or another tile gave up.
constexpr int kProbePerLane = 8;
constexpr int kWindow = 32 * kProbePerLane;

__device__ long long look_back(const EncodeParams &p, const EncodeSmem &sm, long long ticket) {
    const int lane = threadIdx.x & 31;
    const unsigned long long *status = p.ws.tile_status;
    long long base = ticket - 1;  // row q, lane l: word base - 32q - l
    unsigned long long acc = 0;
    unsigned long long t0 = 0;
    unsigned int backoff = 2000;
    bool first_window = true;
    while (true) {
        unsigned long long w[kProbePerLane];
        {
            const long long j = base - lane;
            w[0] = (j >= 0) ? ld_relaxed_gpu(status + j * kStatusStride) : kFlagPrefix;
        }
        int rows = 1;  // rows read so far (1 or kProbePerLane)
        if (!first_window) {
#pragma unroll
            for (int q = 1; q < kProbePerLane; ++q) {
                const long long j = base - 32 * q - lane;
                w[q] = (j >= 0) ? ld_relaxed_gpu(status + j * kStatusStride) : kFlagPrefix;
            }
            rows = kProbePerLane;
        }
        int stop_q, stop_l;  // the nearest prefix-or-unpublished word (stop_q == rows: none)
        bool at_prefix;
        while (true) {
            stop_q = rows;
            stop_l = 0;
            at_prefix = false;
            int pq = rows, pl = 0;  // the nearest prefix word
#pragma unroll
            for (int q = 0; q < kProbePerLane; ++q) {
                if (q < rows && pq == rows) {  // rows past the nearest prefix do not matter
                    const unsigned int f = static_cast<unsigned int>(w[q] >> kFlagShift);
                    const unsigned int pm = __ballot_sync(0xffffffffu, f == 2u);
                    const unsigned int xm = __ballot_sync(0xffffffffu, f == 0u);
                    if (stop_q == rows && (pm | xm) != 0u) {
                        stop_q = q;
                        stop_l = __ffs(pm | xm) - 1;
                        at_prefix = (pm >> stop_l) & 1u;
                    }
                    if (pq == rows && pm != 0u) {
                        pq = q;
                        pl = __ffs(pm) - 1;
                    }
                }
            }
            if (stop_q == rows && rows < kProbePerLane) {
                // the nearest 32 are all aggregates: read the rest of the window
#pragma unroll
                for (int q = 1; q < kProbePerLane; ++q) {
                    const long long j = base - 32 * q - lane;
                    w[q] = (j >= 0) ? ld_relaxed_gpu(status + j * kStatusStride) : kFlagPrefix;
                }
                rows = kProbePerLane;
                continue;
            }
            if (stop_q == rows || at_prefix) break;

            int give_up = 0;
            if (lane == 0) {
                const unsigned long long now = global_timer_ns();
                if (t0 == 0) t0 = now;
                if (now - t0 > static_cast<unsigned long long>(p.wait_limit_ns)) {
                    atomicExch(&p.ws.hdr->abort, 1u);
                    record_error(p.ws.hdr, DWS_ERR_TIMEOUT, ticket);
                    give_up = 1;
                } else if (ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u ||
                           *reinterpret_cast<const volatile int *>(&sm.stop) != 0) {
                    give_up = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, give_up, 0)) return -1;
            __nanosleep(backoff);
            if (backoff < 4000) backoff <<= 1;
#pragma unroll
            for (int q = 0; q < kProbePerLane; ++q) {
                const bool before_p = (q < pq) || (q == pq && lane < pl);
                if (q < rows && before_p && (w[q] >> kFlagShift) == 0ull) {
                    const long long j = base - 32 * q - lane;
                    w[q] = ld_relaxed_gpu(status + j * kStatusStride);
                }
            }
        }
        unsigned long long v = 0;
#pragma unroll
        for (int q = 0; q < kProbePerLane; ++q) {
            const bool take = (q < rows) && (q < stop_q || (q == stop_q && lane <= stop_l));
            if (take) v += w[q] & kValueMask;
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
        acc += v;
        if (stop_q < rows) return static_cast<long long>(acc);  // ended at a prefix
        base -= kWindow;
        first_window = false;
    }
}

// ---------------------------------------------------------------------------
// Producer: lane 0 of warp kProducerWarp
// ---------------------------------------------------------------------------
__device__ void produce(const EncodeParams &p, EncodeSmem &sm) {
    // Lookahead: right after fill k is issued, the ticket of fill k+4 is taken
    // and the descriptor of fill k+2 read (its ticket taken two fills
    // earlier), so neither latency is waited on.
    long long tk0 = take_ticket(p);
    long long tk1 = take_ticket(p);
    long long tk2 = take_ticket(p);
    long long tk3 = take_ticket(p);
    TileDesc dk0 = load_desc(p, tk0);
    TileDesc dk1 = load_desc(p, tk1);
    int markers = 0;
    for (long long k = 0;; ++k) {
        const int s = static_cast<int>(k % kStages);
        if (k >= kStages) {
            const uint32_t parity = static_cast<uint32_t>((k / kStages - 1) & 1);
            unsigned int backoff = 32;
            while (!mbar_try_wait(&sm.empty_bar[s], parity)) {
                if (*reinterpret_cast<volatile int *>(&sm.stop) != 0 ||
                    ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u) {
                    st_release_cta(&sm.producer_done, 1);
                    return;
                }
                __nanosleep(backoff);
                if (backoff < 256) backoff <<= 1;
            }
        }
        if (*reinterpret_cast<volatile int *>(&sm.stop) != 0) break;
        // Issue first: the arrive has release semantics and would otherwise
        // wait for the lookahead loads below to come back.
        issue_stage(p, sm, s, tk0, dk0);
        if (tk0 >= p.ws.num_tiles && ++markers == kGroups) break;  // one end marker per group
        tk0 = tk1;
        tk1 = tk2;
        tk2 = tk3;
        dk0 = dk1;
        dk1 = load_desc(p, tk1);
        tk3 = take_ticket(p);
    }
    st_release_cta(&sm.producer_done, 1);
}

// ---------------------------------------------------------------------------
// Counting groups: group g is threads g * kGroupThreads .. + kGroupThreads - 1
// ---------------------------------------------------------------------------
// A warp whose 1024 elements all changed (a clustered run): each thread's
// 32 entries are its slice itself, read as 16-byte chunks in a rotated,
// bank-conflict-free order, with no bit scan.  Kept out of line so that the
// common path's code is left as it is.
__device__ __noinline__ void dense_slice_to_ring(uint32_t *ring, int rr0, int o0, const uint16_t *new_s,
                                                 int tid) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int cr = (c + (tid >> 1)) & 3;
        const uint4 w = *reinterpret_cast<const uint4 *>(new_s + o0 + 8 * cr);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int k = 8 * cr + 2 * h;
            ring[(rr0 + k) & (kRing - 1)] = static_cast<uint32_t>(o0 + k) | (ww[h] << 16);
            ring[(rr0 + k + 1) & (kRing - 1)] = static_cast<uint32_t>(o0 + k + 1) | (ww[h] & 0xffff0000u);
        }
    }
}

template <bool kCompact>
__device__ void count_group(const EncodeParams &p, EncodeSmem &sm, const int g) {
    const int tid = threadIdx.x - g * kGroupThreads;  // thread within the group
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int bar = kCountBar + g;
    uint32_t *ring = sm.ring[g];

    // The group's thread 0 keeps the group's queue entries (g, g + kGroups,
    // ...) and ring.
    int q_head = g;
    int ring_tail = 0, ring_head = 0;

    long long waits = g;  // the group's next stage fill (fills g, g + kGroups, ...)
    bool failed = false;
    for (;; waits += kGroups) {
        const int s = static_cast<int>(waits % kStages);
        const uint32_t parity = static_cast<uint32_t>((waits / kStages) & 1);
        const bool loaded = mbar_wait(&sm.bar[s], parity, kLoadWaitLimitNs);
        const StageMeta m = sm.meta[s];      // written before the fill's arrive
        const bool done = m.ticket >= p.ws.num_tiles;
        const bool work = loaded && !done;
        const TileDesc &d = m.d;
        if (tid == 0 && work) {
            // A queue slot for this tile (freed in order by the look-back
            // group).  The cached head only lags, so the flags are polled only
            // when the cached view says the queue is full.  Ring space is
            // reserved after the count, for the tile's actual entries.
            unsigned int backoff = 32;
            bool ok = true;
            while (!(waits - q_head < kQueue)) {
                // Plain volatile polling: an acquire would also wait for this
                // thread's outstanding global accesses.  The ring is only
                // rewritten after the flag is seen, and a look-back warp sets
                // its flag after all its ring reads have returned.
                while (q_head < waits &&
                       *reinterpret_cast<volatile int *>(&sm.q_done[q_head % kQueue]) == q_head + 1) {
                    ring_head += kCompact ? sm.q[q_head % kQueue].total : 0;
                    q_head += kGroups;
                }
                if (waits - q_head < kQueue) break;
                if (*reinterpret_cast<volatile int *>(&sm.stop) != 0 ||
                    ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u) {
                    ok = false;
                    break;
                }
                __nanosleep(backoff);
                if (backoff < 1024) backoff <<= 1;
            }
            sm.alloc_pos[g] = ok ? ring_tail : -1;
            sm.ring_free[g] = kRing - (ring_tail - ring_head);
        }

        uint16_t *old_s = sm.buf[s][0];
        uint16_t *new_s = sm.buf[s][1];
        uint32_t mask = 0;  // elements 32 tid + [0, 32)
        if (work) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int slot = ((tid >> 1) + j) & 3;  // conflict-free 16-byte reads
                const int e0 = (4 * tid + slot) * 8;
                uint4 a, b;
                if (e0 + 8 <= d.bulk) {
                    a = *reinterpret_cast<const uint4 *>(old_s + e0);
                    b = *reinterpret_cast<const uint4 *>(new_s + e0);
                } else {
                    uint16_t av[8], bv[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = e0 + q;
                        av[q] = (e < d.count) ? d.old_p[e] : uint16_t(0);
                        bv[q] = (e < d.count) ? d.new_p[e] : uint16_t(0);
                        if (kCompact && e < d.count) new_s[e] = bv[q];
                    }
                    a.x = av[0] | (uint32_t(av[1]) << 16);
                    a.y = av[2] | (uint32_t(av[3]) << 16);
                    a.z = av[4] | (uint32_t(av[5]) << 16);
                    a.w = av[6] | (uint32_t(av[7]) << 16);
                    b.x = bv[0] | (uint32_t(bv[1]) << 16);
                    b.y = bv[2] | (uint32_t(bv[3]) << 16);
                    b.z = bv[4] | (uint32_t(bv[5]) << 16);
                    b.w = bv[6] | (uint32_t(bv[7]) << 16);
                }
                const uint32_t x0 = a.x ^ b.x, x1 = a.y ^ b.y, x2 = a.z ^ b.z, x3 = a.w ^ b.w;
                const uint32_t bits8 = ((x0 & 0xffffu) != 0) | (((x0 >> 16) != 0) << 1) |
                                       (((x1 & 0xffffu) != 0) << 2) | (((x1 >> 16) != 0) << 3) |
                                       (((x2 & 0xffffu) != 0) << 4) | (((x2 >> 16) != 0) << 5) |
                                       (((x3 & 0xffffu) != 0) << 6) | (((x3 >> 16) != 0) << 7);
                mask |= bits8 << (8 * slot);
            }
        }
        const int cnt = __popc(mask);
        int incl = cnt;
#pragma unroll
        for (int dd = 1; dd < 32; dd <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, dd);
            if (lane >= dd) incl += v;
        }
        if (lane == 31) sm.warp_sum[g][warp] = incl;
        // (A) warp sums and ring position visible.  If a load wait ran out
        // anywhere, or a look-back gave up, the group leaves together; a fill
        // whose wait ran out is still pending and is drained below.
        const bool go = loaded && (*reinterpret_cast<volatile int *>(&sm.stop) == 0);
        if (!named_bar_and(bar, kGroupThreads, go)) {
            if (!loaded) record_error(p.ws.hdr, DWS_ERR_TIMEOUT, waits);
            if (loaded) waits += kGroups;
            failed = true;
            break;
        }
        if (done) {  // every thread saw the same loaded meta
            waits += kGroups;
            break;
        }
        const int pos = sm.alloc_pos[g];
        if (pos < 0) {
            waits += kGroups;
            failed = true;
            break;
        }
        int warp_off = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kGroupWarps; ++w) {
            const int v = sm.warp_sum[g][w];
            warp_off += (w < warp) ? v : 0;
            total += v;
        }
        // The count is published at once, before any wait for ring space:
        // every later tile's look-back, on every SM, may be waiting for it,
        // and the rings those look-backs would drain are what this tile may
        // be waiting for.  Published by a thread that does no shared-memory
        // release afterwards (a release would wait for this global store).
        if (tid == kPublishThread && m.ticket != p.withhold) {
            const unsigned long long flag = (m.ticket == 0) ? kFlagPrefix : kFlagAggregate;
            st_relaxed_gpu(p.ws.tile_status + m.ticket * kStatusStride, flag | static_cast<unsigned long long>(total));
        }
        // Room in the ring for this tile's entries: known free space first,
        // else thread 0 polls the flags until the look-back group has
        // written out enough older tiles.
        if (kCompact && total > sm.ring_free[g]) {  // uniform: all read the same words
            if (tid == 0) {
                unsigned int backoff = 32;
                while (kRing - (ring_tail - ring_head) < total) {
                    while (q_head < waits &&
                           *reinterpret_cast<volatile int *>(&sm.q_done[q_head % kQueue]) == q_head + 1) {
                        ring_head += sm.q[q_head % kQueue].total;
                        q_head += kGroups;
                    }
                    if (kRing - (ring_tail - ring_head) >= total) break;
                    if (*reinterpret_cast<volatile int *>(&sm.stop) != 0 ||
                        ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u) {
                        sm.alloc_pos[g] = -1;
                        break;
                    }
                    __nanosleep(backoff);
                    if (backoff < 1024) backoff <<= 1;
                }
            }
            named_bar(bar, kGroupThreads);  // (B) ring space for this tile
            if (sm.alloc_pos[g] < 0) {
                waits += kGroups;
                failed = true;
                break;
            }
        }
        if (kCompact && __all_sync(0xffffffffu, mask == 0xffffffffu)) {
            dense_slice_to_ring(ring, pos + warp_off + incl - cnt, kElemsPerThread * tid, new_s, tid);
        } else if (kCompact) {
            int rr = pos + warp_off + incl - cnt;
            uint32_t mm = mask;
            while (mm) {
                const int bit = __ffs(mm) - 1;
                mm &= mm - 1;
                const int o = kElemsPerThread * tid + bit;
                ring[rr & (kRing - 1)] = static_cast<uint32_t>(o) | (static_cast<uint32_t>(new_s[o]) << 16);
                ++rr;
            }
        }
        named_bar(bar, kGroupThreads);  // (C) entries in the ring, stage s consumed
        if (tid == 0) {
            const int slot = static_cast<int>(waits % kQueue);
            Pending &e = sm.q[slot];
            e.ticket = m.ticket;
            e.tensor = d.tensor;
            e.local_start = d.local_start;
            e.group = g;
            e.pos = pos;
            e.total = total;
            ring_tail += kCompact ? total : 0;
            st_release_cta(&sm.q_ready[slot], static_cast<int>(waits) + 1);
            mbar_arrive(&sm.empty_bar[s]);  // the producer may refill stage s
        }
    }

    // Counting is over: the look-back group stops after the last tile.  The
    // end markers are fills N and N + 1 (one per group), N tiles.
    if (tid == 0 && !failed) atomicMin(&sm.q_final, static_cast<int>(waits - kGroups));
    if (failed) {
        // Leaving on an error: stop the producer, then wait for every fill it
        // issued that has not been consumed.  (A ticket taken but never
        // loaded only happens here, after the global abort flag was set.)
        if (tid == 0) *reinterpret_cast<volatile int *>(&sm.stop) = 1;
        unsigned long long t0 = global_timer_ns();
        while (ld_acquire_cta(&sm.producer_done) == 0 && global_timer_ns() - t0 < kLoadWaitLimitNs) {
            __nanosleep(256);
        }
        named_bar(bar, kGroupThreads);
        for (int k = g; k < kStages; k += kGroups) {  // the group's stages
            // fills of stage k consumed so far (fills before `waits`)
            const long long consumed = (waits + kStages - 1 - k) / kStages;
            if (sm.fills[k] > consumed) {
                mbar_wait(&sm.bar[k], static_cast<uint32_t>(consumed & 1), kLoadWaitLimitNs);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Look-back group: warps kCountWarps .. kCountWarps + kLookWarps - 1
// ---------------------------------------------------------------------------
// The tile's entries, from the ring to indices[prefix ..] and values[prefix ..]
// (those below capacity).  Consecutive lanes store consecutive entries; when
// the outputs are aligned, each lane stores four entries at once (16 bytes of
// indices, 8 of values) after a head that brings the position to a multiple
// of four.
// kWide: int64 global positions, index_base[tensor] + local index.
// kSum: also XOR the written entries into the wire checksum halves (the
// bytes of each position at its tensor's pos_width, the double bits of each
// value) kept in *hp / *hv.
// A look-back lane's share of the wire checksum (kSum).  pos: XOR of the
// positions it wrote; the position hash is the XOR of their bytes at their
// tensor's width, and a 2-byte position (numel <= 65536) has zero upper
// bytes, so folding pos's four bytes at the end gives it for both widths.
// sm, ex: XOR of the sign and mantissa bits, and of e + 896, of the normal
// values (the double's three disjoint fields: sign << 63 | (e + 896) << 52 |
// m << 45); hv: the exact double bits of the other values.
struct SumAcc {
    uint32_t pos, sm, ex;
    unsigned long long hv;
};

template <bool kWide, bool kSum>
__device__ void write_entries(const EncodeParams &p, const uint32_t *ring, const Pending &e,
                              long long prefix, SumAcc *acc) {
    const int lane = threadIdx.x & 31;
    long long lim = p.capacity - prefix;
    if (lim > e.total) lim = e.total;
    const int n = lim > 0 ? static_cast<int>(lim) : 0;
    const uint32_t ls = static_cast<uint32_t>(e.local_start);
    long long gs = 0;  // global position of the tile's first element
    if (kWide) gs = p.index_base[e.tensor] + e.local_start;
    auto sum = [&](uint32_t v) {
        if (kSum) {
            acc->pos ^= ls + (v & 0xffffu);
            const uint32_t b = v >> 16, ee = (b >> 7) & 0xffu;
            if (ee - 1u < 254u) {
                acc->sm ^= b & 0x807fu;
                acc->ex ^= ee + 896u;
            } else {
                acc->hv ^= bf16_to_f64_bits(b);
            }
        }
    };
    auto one = [&](int k) {
        const uint32_t v = ring[(e.pos + k) & (kRing - 1)];
        sum(v);
        if (kWide) {
            st_stream_u64(p.indices64 + prefix + k, static_cast<unsigned long long>(gs + (v & 0xffffu)));
        } else {
            st_stream_u32(p.indices + prefix + k, ls + (v & 0xffffu));
        }
        st_stream_u16(p.values + prefix + k, static_cast<uint16_t>(v >> 16));
    };
    if (!p.vec_out) {
        for (int k = lane; k < n; k += 32) one(k);
        return;
    }
    const int head = static_cast<int>((4 - (prefix & 3)) & 3) < n ? static_cast<int>((4 - (prefix & 3)) & 3) : n;
    if (lane < head) one(lane);
    const int groups = (n - head) >> 2;
    for (int gi = lane; gi < groups; gi += 32) {
        const int k = head + 4 * gi;
        const uint32_t v0 = ring[(e.pos + k) & (kRing - 1)];
        const uint32_t v1 = ring[(e.pos + k + 1) & (kRing - 1)];
        const uint32_t v2 = ring[(e.pos + k + 2) & (kRing - 1)];
        const uint32_t v3 = ring[(e.pos + k + 3) & (kRing - 1)];
        sum(v0);
        sum(v1);
        sum(v2);
        sum(v3);
        if (kWide) {
            st_stream_v2u64(p.indices64 + prefix + k, static_cast<unsigned long long>(gs + (v0 & 0xffffu)),
                            static_cast<unsigned long long>(gs + (v1 & 0xffffu)));
            st_stream_v2u64(p.indices64 + prefix + k + 2, static_cast<unsigned long long>(gs + (v2 & 0xffffu)),
                            static_cast<unsigned long long>(gs + (v3 & 0xffffu)));
        } else {
            st_stream_v4(p.indices + prefix + k,
                         make_uint4(ls + (v0 & 0xffffu), ls + (v1 & 0xffffu), ls + (v2 & 0xffffu),
                                    ls + (v3 & 0xffffu)));
        }
        st_stream_v2(p.values + prefix + k,
                     make_uint2((v0 >> 16) | (v1 & 0xffff0000u), (v2 >> 16) | (v3 & 0xffff0000u)));
    }
    const int tail = head + 4 * groups;
    if (lane < n - tail) one(tail + lane);
}

template <bool kCompact, bool kWide, bool kSum>
__device__ void look_group(const EncodeParams &p, EncodeSmem &sm) {
    const int lane = threadIdx.x & 31;
    const int j = (threadIdx.x >> 5) - kCountWarps;
    SumAcc acc{0u, 0u, 0u, 0ull};  // this lane's share of the checksum (kSum)
    // Leaves through here: the warp's checksum share goes out with one
    // atomic per half (per-tile atomics on two words would be a hot spot).
    auto leave = [&]() {
        if (kSum) {
            const uint32_t x = acc.pos ^ (acc.pos >> 16);
            unsigned long long hp = (x ^ (x >> 8)) & 0xffu;
            unsigned long long hv = acc.hv ^ (static_cast<unsigned long long>((acc.sm >> 15) & 1u) << 63) ^
                                    (static_cast<unsigned long long>(acc.ex & 0x7ffu) << 52) ^
                                    (static_cast<unsigned long long>(acc.sm & 0x7fu) << 45);
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                hp ^= __shfl_xor_sync(0xffffffffu, hp, d);
                hv ^= __shfl_xor_sync(0xffffffffu, hv, d);
            }
            if (lane == 0) {
                if (hp) atomicXor(p.hashes, hp);
                if (hv) atomicXor(p.hashes + 1, hv);
            }
        }
    };
    for (int i = j;; i += kLookWarps) {
        // Wait for queue entry i, or for the end.
        unsigned int backoff = 32;
        for (;;) {
            if (ld_acquire_cta(&sm.q_ready[i % kQueue]) == i + 1) break;
            const int fin = ld_acquire_cta(&sm.q_final);
            if (i >= fin || *reinterpret_cast<volatile int *>(&sm.stop) != 0) {
                leave();
                return;
            }
            __nanosleep(backoff);
            if (backoff < 512) backoff <<= 1;
        }
        const Pending e = sm.q[i % kQueue];
        long long prefix;
        if (e.ticket == p.withhold) {
            prefix = -1;
        } else if (e.ticket == 0) {
            prefix = 0;
        } else {
            prefix = look_back(p, sm, e.ticket);
        }
        if (prefix >= 0) {
            if (lane == 0) {
                if (e.ticket != 0)
                    st_relaxed_gpu(p.ws.tile_status + e.ticket * kStatusStride,
                                   kFlagPrefix | static_cast<unsigned long long>(prefix + e.total));
                if (e.local_start == 0) p.offsets[e.tensor] = prefix;
                if (e.ticket == p.ws.num_tiles - 1) {
                    const long long nnz = prefix + e.total;
                    p.offsets[p.ws.num_tensors] = nnz;
                    if (kCompact && nnz > p.capacity) record_error(p.ws.hdr, DWS_ERR_CAPACITY, nnz);
                }
            }
            if (kCompact) write_entries<kWide, kSum>(p, sm.ring[e.group], e, prefix, &acc);
        } else if (e.ticket != p.withhold) {
            if (lane == 0) *reinterpret_cast<volatile int *>(&sm.stop) = 1;
        }
        // Every lane's ring reads have returned (their values were stored), so
        // a plain store lets the counting group reuse the ring space.
        __syncwarp();
        if (lane == 0) *reinterpret_cast<volatile int *>(&sm.q_done[i % kQueue]) = i + 1;
    }
}

template <bool kCompact, bool kWide, bool kSum>
__global__ void __launch_bounds__(kThreads, 1) encode_kernel(EncodeParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncodeSmem &sm = *reinterpret_cast<EncodeSmem *>(smem_raw);
    const int tid = threadIdx.x;

    if (!ws_matches(p.ws)) return;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.bar[s], 1);
            mbar_init(&sm.empty_bar[s], 1);
            sm.fills[s] = 0;
        }
        mbar_fence_init();
        sm.q_final = 0x7fffffff;
        sm.stop = 0;
        sm.producer_done = 0;
        for (int k = 0; k < kQueue; ++k) {
            sm.q_ready[k] = 0;
            sm.q_done[k] = 0;
        }
    }
    __syncthreads();

    const int warp = tid >> 5;
    if (warp < kCountWarps) {
        count_group<kCompact>(p, sm, warp / kGroupWarps);
    } else if (warp < kProducerWarp) {
        look_group<kCompact, kWide, kSum>(p, sm);
    } else if ((tid & 31) == 0) {
        produce(p, sm);
    }
}

// Per call: clear the scan state and describe every tile (pointers into both
// snapshots, count, bulk-copyable prefix), checking the pointer tables.
__global__ void prepare_kernel(WsView ws, const uint16_t *const *old_ptrs,
                               const uint16_t *const *new_ptrs) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         i < ws.num_tiles; i += stride) {
        ws.tile_status[i * kStatusStride] = 0ull;
        TileDesc d;
        d.old_p = nullptr;
        d.new_p = nullptr;
        d.tensor = 0;
        d.local_start = 0;
        d.count = 0;
        d.bulk = 0;
        const int t = ws.tile_tensor[i];
        bool ok = (t >= 0 && t < ws.num_tensors);
        if (ok) {
            const long long n = ws.numel[t];
            const long long ls = (i - ws.first_tile[t]) << kTileShift;
            ok = (ls >= 0 && ls <= n);
            if (ok) {
                const long long rest = n - ls;
                d.tensor = t;
                d.local_start = static_cast<int>(ls);
                d.count = static_cast<int>(rest < kTileElems ? rest : kTileElems);
                if (d.count > 0) {
                    const uint16_t *op = old_ptrs[t];
                    const uint16_t *np = new_ptrs[t];
                    const uintptr_t ua = reinterpret_cast<uintptr_t>(op);
                    const uintptr_t ub = reinterpret_cast<uintptr_t>(np);
                    if (op == nullptr || np == nullptr || ((ua | ub) & 1u)) {
                        record_error(ws.hdr, DWS_ERR_INVALID, t);
                        d.count = 0;
                    } else {
                        d.old_p = op + ls;
                        d.new_p = np + ls;
                        d.bulk = ((ua | ub) & 15u) == 0 ? (d.count & ~7) : 0;
                    }
                }
            }
        }
        if (!ok) record_error(ws.hdr, DWS_ERR_WORKSPACE, i);
        ws.tile_desc[i] = d;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        ws.hdr->ticket = 0ull;
        ws.hdr->abort = 0u;
    }
}

// tile_tensor[i] = the tensor t with first_tile[t] <= i < first_tile[t+1].
__global__ void fill_tile_map_kernel(WsView ws) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    int *map = const_cast<int *>(ws.tile_tensor);
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         i < ws.num_tiles; i += stride) {
        int lo = 0, hi = ws.num_tensors;  // first_tile[lo] <= i < first_tile[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (ws.first_tile[mid] <= i) lo = mid;
            else hi = mid;
        }
        map[i] = lo;
    }
}

}  // namespace

size_t encode_smem_bytes() { return sizeof(EncodeSmem); }

cudaError_t encode_set_attributes() {
    const int bytes = static_cast<int>(sizeof(EncodeSmem));
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<true, false, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(encode_kernel<true, true, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(encode_kernel<true, false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(encode_kernel<false, false, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

cudaError_t encode_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, encode_kernel<true, false, false>,
                                                         kThreads, sizeof(EncodeSmem));
}

cudaError_t launch_fill_tile_map(const WsView &ws, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    long long blocks = (ws.num_tiles + 255) / 256;
    if (blocks > 8LL * di.sm_count) blocks = 8LL * di.sm_count;
    if (blocks < 1) blocks = 1;
    fill_tile_map_kernel<<<static_cast<unsigned int>(blocks), 256, 0, s>>>(ws);
    return launched();
}

cudaError_t launch_encode(const WsView &ws, const uint16_t *const *old_ptrs,
                          const uint16_t *const *new_ptrs, long long *offsets, int *indices,
                          uint16_t *values, long long capacity, bool compact,
                          long long wait_limit_ns, long long withhold_tile, cudaStream_t s,
                          long long *indices64, const long long *index_base,
                          unsigned long long *hashes) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    long long pblocks = (ws.num_tiles + 255) / 256;
    if (pblocks > 8LL * di.sm_count) pblocks = 8LL * di.sm_count;
    if (pblocks < 1) pblocks = 1;
    prepare_kernel<<<static_cast<unsigned int>(pblocks), 256, 0, s>>>(ws, old_ptrs, new_ptrs);
    e = launched();
    if (e != cudaSuccess) return e;

    EncodeParams p;
    p.ws = ws;
    p.offsets = offsets;
    p.indices = indices;
    p.values = values;
    p.capacity = compact ? capacity : 0;
    p.wait_limit_ns = wait_limit_ns > 0 ? wait_limit_ns : 2000000000LL;
    p.withhold = withhold_tile;
    p.indices64 = indices64;
    p.index_base = index_base;
    p.hashes = hashes;
    if (hashes != nullptr) {
        e = cudaMemsetAsync(hashes, 0, 2 * sizeof(unsigned long long), s);
        if (e != cudaSuccess) return e;
    }
    const uintptr_t ia = indices64 != nullptr ? reinterpret_cast<uintptr_t>(indices64)
                                              : reinterpret_cast<uintptr_t>(indices);
    p.vec_out = ((ia & 15u) == 0 && (reinterpret_cast<uintptr_t>(values) & 7u) == 0) ? 1 : 0;

    long long grid = static_cast<long long>(di.sm_count) * di.encode_ctas_per_sm;
    if (grid > ws.num_tiles) grid = ws.num_tiles;
    if (grid < 1) grid = 1;
    const size_t smem = sizeof(EncodeSmem);
    if (compact) {
        if (indices64 != nullptr) {
            encode_kernel<true, true, false><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
        } else if (hashes != nullptr) {
            encode_kernel<true, false, true><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
        } else {
            encode_kernel<true, false, false><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
        }
    } else {
        encode_kernel<false, false, false><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
    }
    return launched();
}

}  // namespace dws
