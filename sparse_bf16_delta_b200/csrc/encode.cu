// encode.cu -- fused change detection, scan and compaction (one launch).
//
// What it computes ([verl] review, key source snippets, sparse_gather.py,
// shard_delta_indices; "Delta Weight Sync in TRL" §4.1/§4.2): for every
// tensor of the plan, the ascending local indices i where the 16-bit pattern
// of new[i] differs from old[i], and new[i] at those indices, concatenated in
// plan order with a per-tensor offsets[] prefix.
//
// How (single pass over both snapshots, 4 bytes read per element):
//   * Persistent CTAs take tiles (8192 elements) by atomic ticket, so a tile's
//     predecessors are always resident or finished (forward progress of the
//     scan below).
//   * Each CTA keeps kStages tiles in flight: thread 0 issues 1-D bulk async
//     copies (cp.async.bulk, global -> own shared memory, mbarrier
//     transaction counts, L2 evict-first) of both snapshots for the next
//     tickets while the CTA works on the current one.
//   * detect: 16-byte shared-memory reads in a bank-conflict-free order, a
//     32-bit change mask per thread, popc; block scan of the counts.
//   * scan: decoupled look-back over the tile status words (flag + 62-bit
//     count), a warp probing 32 predecessors at a time; bounded by a wall-clock
//     limit after which the kernel records DWS_ERR_TIMEOUT and all waiters
//     leave.
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

constexpr unsigned long long kLoadWaitLimitNs = 4000000000ull;  // 4 s

struct StageMeta {
    long long ticket;      // >= num_tiles: no more work
    const uint16_t *old_p;  // tile start in the old snapshot
    const uint16_t *new_p;  // tile start in the new snapshot
    int tensor;
    int local_start;  // first element of the tile within its tensor
    int count;        // elements in the tile (0 .. kTileElems)
    int bulk;         // leading elements delivered by bulk copy (multiple of 8)
};

struct EncodeParams {
    WsView ws;
    const uint16_t *const *old_ptrs;
    const uint16_t *const *new_ptrs;
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
    int warp_sum[kWarps];
    long long tile_prefix;
};

// Thread 0: take the next ticket and start loading it into stage s.
__device__ void issue_tile(const EncodeParams &p, EncodeSmem &sm, int s,
                           unsigned long long policy) {
    StageMeta m;
    m.ticket = static_cast<long long>(atomicAdd(&p.ws.hdr->ticket, 1ull));
    m.old_p = nullptr;
    m.new_p = nullptr;
    m.tensor = 0;
    m.local_start = 0;
    m.count = 0;
    m.bulk = 0;
    if (m.ticket < p.ws.num_tiles) {
        const int t = p.ws.tile_tensor[m.ticket];
        bool ok = (t >= 0 && t < p.ws.num_tensors);
        if (ok) {
            const long long first = p.ws.first_tile[t];
            const long long n = p.ws.numel[t];
            const long long ls = (m.ticket - first) << kTileShift;
            ok = (ls >= 0 && ls <= n);
            if (ok) {
                const long long rest = n - ls;
                m.tensor = t;
                m.local_start = static_cast<int>(ls);
                m.count = static_cast<int>(rest < kTileElems ? rest : kTileElems);
                if (m.count > 0) {
                    const uint16_t *op = p.old_ptrs[t];
                    const uint16_t *np = p.new_ptrs[t];
                    const uintptr_t ua = reinterpret_cast<uintptr_t>(op);
                    const uintptr_t ub = reinterpret_cast<uintptr_t>(np);
                    if (op == nullptr || np == nullptr || ((ua | ub) & 1u)) {
                        record_error(p.ws.hdr, DWS_ERR_INVALID, t);
                        m.count = 0;
                    } else {
                        m.old_p = op + ls;
                        m.new_p = np + ls;
                        m.bulk = ((ua | ub) & 15u) == 0 ? (m.count & ~7) : 0;
                    }
                }
            }
        }
        if (!ok) {
            record_error(p.ws.hdr, DWS_ERR_WORKSPACE, m.ticket);
            m.count = 0;
        }
        mbar_arrive_expect_tx(&sm.bar[s], static_cast<uint32_t>(m.bulk) * 4u);
        if (m.bulk > 0) {
            const uint32_t bytes = static_cast<uint32_t>(m.bulk) * 2u;
            bulk_load(sm.buf[s][0], m.old_p, bytes, &sm.bar[s], policy);
            bulk_load(sm.buf[s][1], m.new_p, bytes, &sm.bar[s], policy);
        }
    }
    sm.meta[s] = m;
}

// Warp 0: exclusive prefix of tile `ticket` by decoupled look-back.
// Returns -1 if the bounded wait ran out or another tile gave up.
__device__ long long look_back(const EncodeParams &p, long long ticket) {
    const int lane = threadIdx.x & 31;
    unsigned long long *status = p.ws.tile_status;
    long long base = ticket - 1;
    unsigned long long acc = 0;
    unsigned long long t0 = 0;
    unsigned int backoff = 32;
    while (true) {
        const long long j = base - lane;
        const unsigned long long st = (j >= 0) ? ld_relaxed_gpu(status + j) : kFlagPrefix;
        const unsigned int flag = static_cast<unsigned int>(st >> kFlagShift);
        const unsigned int pmask = __ballot_sync(0xffffffffu, flag == 2u);
        const unsigned int xmask = __ballot_sync(0xffffffffu, flag == 0u);
        const int first_p = pmask ? (__ffs(pmask) - 1) : 32;
        const unsigned int needed = (first_p >= 31) ? 0xffffffffu : ((2u << first_p) - 1u);
        if (xmask & needed) {
            // Some predecessor has not published yet: wait, boundedly.
            int give_up = 0;
            if (lane == 0) {
                const unsigned long long now = global_timer_ns();
                if (t0 == 0) t0 = now;
                if (now - t0 > static_cast<unsigned long long>(p.wait_limit_ns)) {
                    atomicExch(&p.ws.hdr->abort, 1u);
                    record_error(p.ws.hdr, DWS_ERR_TIMEOUT, ticket);
                    give_up = 1;
                } else if (ld_relaxed_gpu_u32(&p.ws.hdr->abort) != 0u) {
                    give_up = 1;
                }
            }
            give_up = __shfl_sync(0xffffffffu, give_up, 0);
            if (give_up) return -1;
            __nanosleep(backoff);
            if (backoff < 1024) backoff <<= 1;
            continue;
        }
        unsigned long long v = (lane <= first_p) ? (st & kValueMask) : 0ull;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
        acc += v;
        if (first_p < 32) return static_cast<long long>(acc);
        base -= 32;
    }
}

template <bool kCompact>
__global__ void __launch_bounds__(kThreads, 2) encode_kernel(EncodeParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncodeSmem &sm = *reinterpret_cast<EncodeSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (!ws_matches(p.ws)) return;

    unsigned long long policy = 0;
    if (tid == 0) {
        policy = l2_evict_first_policy();
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[s], 1);
        mbar_fence_init();
        for (int s = 0; s < kStages; ++s) issue_tile(p, sm, s, policy);
    }
    __syncthreads();

    uint32_t phase_bits = 0;
    bool stop = false;
    int s = 0;
    for (;;) {
        const StageMeta m = sm.meta[s];
        if (m.ticket >= p.ws.num_tiles) break;

        // ---- wait for the tile's bulk copies -------------------------------
        const uint32_t parity = (phase_bits >> s) & 1u;
        phase_bits ^= (1u << s);
        const bool loaded = mbar_wait(&sm.bar[s], parity, kLoadWaitLimitNs);

        uint16_t *old_s = sm.buf[s][0];
        uint16_t *new_s = sm.buf[s][1];

        // ---- detect: 32 elements per thread, 4 chunks of 8 ----------------
        uint32_t mask = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int slot = ((tid >> 1) + j) & 3;  // conflict-free 16-byte reads
            const int c = 4 * tid + slot;
            const int e0 = c * 8;
            uint4 a, b;
            if (e0 + 8 <= m.bulk) {
                a = *reinterpret_cast<const uint4 *>(old_s + e0);
                b = *reinterpret_cast<const uint4 *>(new_s + e0);
            } else {
                uint16_t av[8], bv[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int e = e0 + q;
                    av[q] = (e < m.count) ? m.old_p[e] : uint16_t(0);
                    bv[q] = (e < m.count) ? m.new_p[e] : uint16_t(0);
                    if (kCompact && e < m.count) new_s[e] = bv[q];
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
            uint32_t bits8 = ((x0 & 0xffffu) != 0) | (((x0 >> 16) != 0) << 1) |
                             (((x1 & 0xffffu) != 0) << 2) | (((x1 >> 16) != 0) << 3) |
                             (((x2 & 0xffffu) != 0) << 4) | (((x2 >> 16) != 0) << 5) |
                             (((x3 & 0xffffu) != 0) << 6) | (((x3 >> 16) != 0) << 7);
            mask |= bits8 << (8 * slot);
        }
        const int cnt = __popc(mask);

        // ---- block scan of the per-thread counts --------------------------
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += v;
        }
        if (lane == 31) sm.warp_sum[warp] = incl;
        // (1) counts published; everyone is done reading old_s.  The load wait
        // is bounded; if it ran out anywhere, the whole CTA leaves together
        // before anything is published or written.
        if (!__syncthreads_and(loaded)) {
            if (tid == 0) record_error(p.ws.hdr, DWS_ERR_TIMEOUT, m.ticket);
            return;
        }
        int warp_off = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int v = sm.warp_sum[w];
            warp_off += (w < warp) ? v : 0;
            total += v;
        }
        const int excl = warp_off + incl - cnt;

        // Warp 0 publishes the tile's aggregate before anything else.
        const bool withheld = (m.ticket == p.withhold);
        if (tid == 0 && !withheld) {
            const unsigned long long flag = (m.ticket == 0) ? kFlagPrefix : kFlagAggregate;
            st_relaxed_gpu(p.ws.tile_status + m.ticket,
                           flag | static_cast<unsigned long long>(total));
        }

        // ---- stage the changed offsets (in ascending order) ---------------
        if (kCompact) {
            uint16_t *stage = old_s;
            uint32_t mm = mask;
            int r = excl;
            while (mm) {
                const int bit = __ffs(mm) - 1;
                mm &= mm - 1;
                stage[r++] = static_cast<uint16_t>(32 * tid + bit);
            }
        }

        // ---- scan: exclusive prefix of this tile --------------------------
        if (warp == 0) {
            long long prefix;
            if (withheld) {
                prefix = -1;
            } else if (m.ticket == 0) {
                prefix = 0;
            } else {
                prefix = look_back(p, m.ticket);
                if (lane == 0 && prefix >= 0) {
                    st_relaxed_gpu(p.ws.tile_status + m.ticket,
                                   kFlagPrefix | static_cast<unsigned long long>(prefix + total));
                }
            }
            if (lane == 0) sm.tile_prefix = prefix;
        }
        __syncthreads();  // (2) staging complete, prefix known
        const long long prefix = sm.tile_prefix;

        if (prefix >= 0) {
            if (tid == 0) {
                if (m.local_start == 0) p.offsets[m.tensor] = prefix;
                if (m.ticket == p.ws.num_tiles - 1) {
                    const long long nnz = prefix + total;
                    p.offsets[p.ws.num_tensors] = nnz;
                    if (kCompact && nnz > p.capacity) record_error(p.ws.hdr, DWS_ERR_CAPACITY, nnz);
                }
            }
            // ---- compact: coalesced writes of the staged entries ----------
            if (kCompact) {
                const uint16_t *stage = old_s;
                for (int i = tid; i < total; i += kThreads) {
                    const long long pos = prefix + i;
                    if (pos < p.capacity) {
                        const int o = stage[i];
                        st_stream_u32(p.indices + pos, static_cast<uint32_t>(m.local_start + o));
                        st_stream_u16(p.values + pos, new_s[o]);
                    }
                }
            }
        } else if (!withheld) {
            stop = true;  // the scan gave up: nothing after this tile is valid
        }
        __syncthreads();  // (3) stage s fully consumed

        if (stop) break;
        if (tid == 0) issue_tile(p, sm, s, policy);
        s = (s + 1 == kStages) ? 0 : s + 1;
    }

    // Leaving early: wait for the loads still in flight into our buffers.
    if (stop) {
        for (int k = 1; k < kStages; ++k) {
            const int t = (s + k) % kStages;
            if (sm.meta[t].ticket < p.ws.num_tiles) {
                const uint32_t parity = (phase_bits >> t) & 1u;
                mbar_wait(&sm.bar[t], parity, kLoadWaitLimitNs);
            }
        }
    }
}

__global__ void ws_reset_kernel(WsView ws) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         i < ws.num_tiles; i += stride) {
        ws.tile_status[i] = 0ull;
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

cudaError_t launch_ws_reset(const WsView &ws, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    long long blocks = (ws.num_tiles + 255) / 256;
    if (blocks > 4LL * di.sm_count) blocks = 4LL * di.sm_count;
    if (blocks < 1) blocks = 1;
    ws_reset_kernel<<<static_cast<unsigned int>(blocks), 256, 0, s>>>(ws);
    return launched();
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
    e = launch_ws_reset(ws, s);
    if (e != cudaSuccess) return e;

    EncodeParams p;
    p.ws = ws;
    p.old_ptrs = old_ptrs;
    p.new_ptrs = new_ptrs;
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
