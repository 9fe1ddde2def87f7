// apply.cu -- receiver side: scatter one delta onto a snapshot, in place
// ("Delta Weight Sync in TRL" §4.3 receive_weights: for each tensor t and
// entry j of its segment, snap_t[indices[j]] = values[j]), and the checks of
// a delta's offsets that every delta consumer runs first.
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
// The replay of a chain of deltas is in chain.cu.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

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

}  // namespace

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

}  // namespace dws
