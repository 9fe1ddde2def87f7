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
//   * Persistent CTAs (256 threads, 2 per SM) take tiles of 8192 elements by
//     atomic ticket, so a tile's predecessors are always resident or finished
//     (forward progress of the scan below).  Each CTA owns kStages stages,
//     each holding both snapshots' 16 KiB of a tile, filled by two 1-D bulk
//     async copies (cp.async.bulk, global -> own shared memory, mbarrier
//     transaction count, L2 evict-first).
//   * The CTA runs an event loop that never blocks on the scan.  Each turn it
//     (a) counts the oldest loaded stage if its data has arrived --
//     detect, block scan, publish the tile's count, stage the changed offsets
//     -- and (b) takes one non-blocking look-back step for the oldest counted
//     tile; when that tile's prefix is known it writes the tile's entries,
//     and the freed stage is refilled with a new ticket.  A tile's count thus
//     depends only on its own data arriving, never on another tile's
//     look-back: a ticket that is held while its CTA waits on a look-back
//     makes every later tile wait on it in turn (convoys).
//   * detect: 16-byte shared-memory reads in a bank-conflict-free order, a
//     32-bit change mask per thread, popc; block scan of the counts.
//   * scan: decoupled look-back over the tile status words (flag + 62-bit
//     count); warp 0 reads 256 predecessors per round trip (8 per lane) and,
//     while waiting, re-reads only the words still unpublished (re-reading
//     whole windows from every waiting warp floods the L2 with requests to
//     the hottest lines).  Bounded by a wall-clock limit after which the
//     kernel records DWS_ERR_TIMEOUT and every CTA leaves.
//   * compact: the tile's changed offsets are staged in shared memory (over
//     the old snapshot's slot, no longer needed), then written out with
//     consecutive threads storing consecutive entries (coalesced).
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 3;
constexpr int kChunks = kTileElems / 8;  // 16-byte chunks of bf16 per tile
static_assert(kChunks == 4 * kThreads, "each thread owns 4 chunks (32 elements)");

// Stage states.
constexpr int kEmptyDone = 0;  // no more tickets for this stage
constexpr int kLoading = 1;    // ticket taken, bulk copies in flight
constexpr int kCounted = 2;    // count published, waiting for its prefix

// Look-back step results.
constexpr long long kNotReady = -2;
constexpr long long kGaveUp = -1;

struct StageMeta {
    long long ticket;
    TileDesc d;
};

struct EncodeParams {
    WsView ws;
    long long *offsets;
    int *indices;
    uint16_t *values;
    long long capacity;
    long long wait_limit_ns;
    long long withhold;
};

struct EncodeSmem {
    uint16_t buf[kStages][2][kTileElems];  // [stage][0 = old | staging, 1 = new]
    unsigned long long bar[kStages];
    StageMeta meta[kStages];
    int state[kStages];
    int total[kStages];
    int warp_sum[kWarps];
    long long step_result;
};

// Thread 0: take the next ticket, read its descriptor, start loading it into
// stage s (or mark the stage done).
__device__ void refill(const EncodeParams &p, EncodeSmem &sm, int s) {
    StageMeta m;
    m.ticket = static_cast<long long>(atomicAdd(&p.ws.hdr->ticket, 1ull));
    if (m.ticket < p.ws.num_tiles) {
        m.d = p.ws.tile_desc[m.ticket];
        const uint32_t bulk = static_cast<uint32_t>(m.d.bulk);
        mbar_arrive_expect_tx(&sm.bar[s], bulk * 4u);
        if (bulk > 0) {
            const unsigned long long policy = l2_evict_first_policy();
            bulk_load(sm.buf[s][0], m.d.old_p, bulk * 2u, &sm.bar[s], policy);
            bulk_load(sm.buf[s][1], m.d.new_p, bulk * 2u, &sm.bar[s], policy);
        }
        sm.state[s] = kLoading;
    } else {
        sm.state[s] = kEmptyDone;
    }
    sm.meta[s] = m;
}

// Resumable decoupled look-back, run by warp 0 (state in its registers).
// Lane l holds predecessors base - 8l - q (q = 0..7, newest first).
constexpr int kProbePerLane = 8;
constexpr int kWindow = 32 * kProbePerLane;

struct LookBack {
    long long ticket;
    long long base;
    unsigned long long acc;
    unsigned long long t0;
    unsigned long long w[kProbePerLane];
};

__device__ __forceinline__ void lb_load_window(LookBack &lb, const unsigned long long *status) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < kProbePerLane; ++q) {
        const long long j = lb.base - kProbePerLane * lane - q;
        lb.w[q] = (j >= 0) ? ld_relaxed_gpu(status + j) : kFlagPrefix;
    }
}

__device__ __forceinline__ void lb_start(LookBack &lb, const EncodeParams &p, long long ticket) {
    lb.ticket = ticket;
    lb.base = ticket - 1;
    lb.acc = 0;
    lb.t0 = 0;
    lb_load_window(lb, p.ws.tile_status);
}

// One step: evaluate the window loaded by the previous step.  Returns the
// exclusive prefix, kNotReady (loads for the next step issued), or kGaveUp.
__device__ long long lb_step(LookBack &lb, const EncodeParams &p) {
    const int lane = threadIdx.x & 31;
    int first_p = kProbePerLane;
    bool unready = false;
    unsigned long long sum = 0;
#pragma unroll
    for (int q = 0; q < kProbePerLane; ++q) {
        if (first_p == kProbePerLane) {
            const unsigned int flag = static_cast<unsigned int>(lb.w[q] >> kFlagShift);
            if (flag == 0u) {
                unready = true;
            } else {
                sum += lb.w[q] & kValueMask;
                if (flag == 2u) first_p = q;
            }
        }
    }
    const unsigned int pmask = __ballot_sync(0xffffffffu, first_p < kProbePerLane);
    const int p_lane = pmask ? (__ffs(pmask) - 1) : 32;
    const bool blocks = (lane <= p_lane) && unready;
    if (__any_sync(0xffffffffu, blocks)) {
        int give_up = 0;
        if (lane == 0) {
            const unsigned long long now = global_timer_ns();
            if (lb.t0 == 0) lb.t0 = now;
            if (now - lb.t0 > static_cast<unsigned long long>(p.wait_limit_ns)) {
                atomicExch(&p.ws.hdr->abort, 1u);
                record_error(p.ws.hdr, DWS_ERR_TIMEOUT, lb.ticket);
                give_up = 1;
            } else if (ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u) {
                give_up = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, give_up, 0)) return kGaveUp;
        // Re-read only the unpublished words that are needed.
        if (blocks) {
#pragma unroll
            for (int q = 0; q < kProbePerLane; ++q) {
                if ((lb.w[q] >> kFlagShift) == 0ull) {
                    const long long j = lb.base - kProbePerLane * lane - q;
                    lb.w[q] = ld_relaxed_gpu(p.ws.tile_status + j);
                }
            }
        }
        return kNotReady;
    }
    unsigned long long v = (lane <= p_lane) ? sum : 0ull;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    lb.acc += v;
    if (p_lane < 32) return static_cast<long long>(lb.acc);
    lb.base -= kWindow;
    lb_load_window(lb, p.ws.tile_status);
    return kNotReady;
}

template <bool kCompact>
__global__ void __launch_bounds__(kThreads, 2) encode_kernel(EncodeParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncodeSmem &sm = *reinterpret_cast<EncodeSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (!ws_matches(p.ws)) return;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[s], 1);
        mbar_fence_init();
        for (int s = 0; s < kStages; ++s) refill(p, sm, s);
    }
    __syncthreads();

    uint32_t phase_bits = 0;
    int next_count = 0;   // oldest stage still to be counted (ring order)
    int next_finish = 0;  // oldest counted stage waiting for its prefix
    bool lb_active = false;
    LookBack lb;
    bool stop = false;

    for (;;) {
        const int fs = next_finish;
        const int f_state = sm.state[fs];
        if (f_state == kEmptyDone) break;  // every stage after it is done too
        bool progress = false;

        // ---- (a) count the oldest loaded stage once its data is there ------
        const int c = next_count;
        if (sm.state[c] == kLoading) {
            const uint32_t parity = (phase_bits >> c) & 1u;
            const bool ready = __syncthreads_and(mbar_try_wait(&sm.bar[c], parity));
            if (ready) {
                phase_bits ^= (1u << c);
                const StageMeta m = sm.meta[c];
                const TileDesc &d = m.d;
                uint16_t *old_s = sm.buf[c][0];
                uint16_t *new_s = sm.buf[c][1];
                uint32_t mask = 0;
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
                    const uint32_t bits8 =
                        ((x0 & 0xffffu) != 0) | (((x0 >> 16) != 0) << 1) |
                        (((x1 & 0xffffu) != 0) << 2) | (((x1 >> 16) != 0) << 3) |
                        (((x2 & 0xffffu) != 0) << 4) | (((x2 >> 16) != 0) << 5) |
                        (((x3 & 0xffffu) != 0) << 6) | (((x3 >> 16) != 0) << 7);
                    mask |= bits8 << (8 * slot);
                }
                const int cnt = __popc(mask);
                int incl = cnt;
#pragma unroll
                for (int dd = 1; dd < 32; dd <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, dd);
                    if (lane >= dd) incl += v;
                }
                if (lane == 31) sm.warp_sum[warp] = incl;
                __syncthreads();  // warp sums visible; old_s no longer read
                int warp_off = 0, total = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const int v = sm.warp_sum[w];
                    warp_off += (w < warp) ? v : 0;
                    total += v;
                }
                if (tid == 0) {
                    if (m.ticket != p.withhold) {
                        const unsigned long long flag =
                            (m.ticket == 0) ? kFlagPrefix : kFlagAggregate;
                        st_relaxed_gpu(p.ws.tile_status + m.ticket,
                                       flag | static_cast<unsigned long long>(total));
                    }
                    sm.total[c] = total;
                    sm.state[c] = kCounted;
                }
                if (kCompact) {
                    uint16_t *stage = old_s;
                    uint32_t mm = mask;
                    int rr = warp_off + incl - cnt;
                    while (mm) {
                        const int bit = __ffs(mm) - 1;
                        mm &= mm - 1;
                        stage[rr++] = static_cast<uint16_t>(32 * tid + bit);
                    }
                }
                next_count = (c + 1 == kStages) ? 0 : c + 1;
                progress = true;
                __syncthreads();  // staging, state and total visible
            }
        }

        // ---- (b) one look-back step for the oldest counted tile ------------
        if (sm.state[fs] == kCounted) {
            const StageMeta m = sm.meta[fs];
            if (warp == 0) {
                long long r;
                if (m.ticket == p.withhold) {
                    r = kGaveUp;
                } else if (m.ticket == 0) {
                    r = 0;
                } else {
                    if (!lb_active) {
                        lb_start(lb, p, m.ticket);
                        lb_active = true;
                    }
                    r = lb_step(lb, p);
                }
                if (lane == 0) {
                    if (r >= 0 && m.ticket != 0) {
                        st_relaxed_gpu(p.ws.tile_status + m.ticket,
                                       kFlagPrefix |
                                           static_cast<unsigned long long>(r + sm.total[fs]));
                    }
                    sm.step_result = r;
                }
                if (r != kNotReady) lb_active = false;
            }
            __syncthreads();
            const long long prefix = sm.step_result;
            if (prefix != kNotReady) {
                const TileDesc &d = m.d;
                const int total = sm.total[fs];
                if (prefix >= 0) {
                    if (tid == 0) {
                        if (d.local_start == 0) p.offsets[d.tensor] = prefix;
                        if (m.ticket == p.ws.num_tiles - 1) {
                            const long long nnz = prefix + total;
                            p.offsets[p.ws.num_tensors] = nnz;
                            if (kCompact && nnz > p.capacity)
                                record_error(p.ws.hdr, DWS_ERR_CAPACITY, nnz);
                        }
                    }
                    if (kCompact) {
                        const uint16_t *stage = sm.buf[fs][0];
                        const uint16_t *new_s = sm.buf[fs][1];
                        for (int i = tid; i < total; i += kThreads) {
                            const long long pos = prefix + i;
                            if (pos < p.capacity) {
                                const int o = stage[i];
                                st_stream_u32(p.indices + pos,
                                              static_cast<uint32_t>(d.local_start + o));
                                st_stream_u16(p.values + pos, new_s[o]);
                            }
                        }
                    }
                } else if (m.ticket != p.withhold) {
                    stop = true;  // the scan gave up: nothing after this tile is valid
                }
                __syncthreads();  // stage fs fully consumed
                if (stop) break;
                if (tid == 0) refill(p, sm, fs);
                next_finish = (fs + 1 == kStages) ? 0 : fs + 1;
                progress = true;
                __syncthreads();  // refilled state visible
            }
        }
        if (!progress) __nanosleep(64);
    }

    // Leaving early: wait for the loads still in flight into our stages.
    if (stop) {
        for (int s = 0; s < kStages; ++s) {
            if (sm.state[s] == kLoading) {
                const uint32_t parity = (phase_bits >> s) & 1u;
                mbar_wait(&sm.bar[s], parity, 4000000000ull);
            }
        }
    }
}

// Per call: clear the scan state and describe every tile (pointers into both
// snapshots, count, bulk-copyable prefix), checking the pointer tables.
__global__ void prepare_kernel(WsView ws, const uint16_t *const *old_ptrs,
                               const uint16_t *const *new_ptrs) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         i < ws.num_tiles; i += stride) {
        ws.tile_status[i] = 0ull;
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
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(EncodeSmem)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(encode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(EncodeSmem)));
}

cudaError_t encode_occupancy(int *ctas_per_sm) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, encode_kernel<true>,
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
                          long long wait_limit_ns, long long withhold_tile, cudaStream_t s) {
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

    long long grid = static_cast<long long>(di.sm_count) * di.encode_ctas_per_sm;
    if (grid > ws.num_tiles) grid = ws.num_tiles;
    if (grid < 1) grid = 1;
    const size_t smem = sizeof(EncodeSmem);
    if (compact) {
        encode_kernel<true><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
    } else {
        encode_kernel<false><<<static_cast<unsigned int>(grid), kThreads, smem, s>>>(p);
    }
    return launched();
}

}  // namespace dws
