// gather.cu -- rank 0's side of gathering sharded deltas ([verl] review of
// PR #6974, key source snippets, sparse_gather.py gather_v_batched_to_rank0):
// every rank has encoded its shard of each parameter with global int64
// positions (dws_encode_global), the per-rank buffers have been gathered to
// rank 0 padded to a common length, and rank 0 splits each by its counts and
// concatenates, per parameter, the ranks' pieces in rank order.
//
// dws_merge_shards does that split-and-concatenate on the device from the
// gathered buffers and the ranks' offsets (a dws delta layout per rank):
//   merge_offsets_kernel  offsets[t] = sum over ranks of rank_offsets[r][t]
//                         (the merged layout needs no scan: the sum of the
//                         ranks' prefixes is the prefix of the sums), after
//                         checking each rank's layout;
//   merge_copy_kernel     every entry j of rank r, tensor t, moves to
//                         offsets[t] + (rank r's predecessors' entries of t)
//                         + (j - rank_offsets[r][t]): a permutation of runs,
//                         read and written with coalesced accesses.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMergePerThread = 8;
constexpr int kMergeEntries = kMergeThreads * kMergePerThread;

struct MergeParams {
    WsView ws;
    int R;
    const long long *rank_offsets;  // [R][T+1]
    const long long *rank_indices;  // rank r's entries at r * stride
    const uint16_t *rank_values;
    long long stride;
    long long *offsets;  // [T+1]
    long long *indices;
    uint16_t *values;
    long long capacity;
};

// Grid-stride over t = 0..T: sums the ranks' offsets and checks every rank's
// layout (starts at 0, non-decreasing, ends within the padded length); a bad
// layout sets the delta flag (the copy then writes nothing) and records
// DWS_ERR_BAD_DELTA with detail = -1 - rank.
__global__ void __launch_bounds__(kMergeThreads) merge_offsets_kernel(MergeParams p) {
    if (!ws_matches(p.ws)) return;
    const int T = p.ws.num_tensors;
    const long long stride_t = static_cast<long long>(T) + 1;
    for (int t = blockIdx.x * kMergeThreads + threadIdx.x; t <= T; t += gridDim.x * kMergeThreads) {
        long long sum = 0;
        for (int r = 0; r < p.R; ++r) {
            const long long *ro = p.rank_offsets + r * stride_t;
            const long long v = ro[t];
            const bool bad = (t == 0 && v != 0) || (t > 0 && v < ro[t - 1]) || (t == T && v > p.stride);
            if (bad) {
                atomicOr(&p.ws.hdr->delta_bad, 1u);
                record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, -1 - static_cast<long long>(r));
            }
            sum += v;
        }
        p.offsets[t] = sum;
        if (t == T && sum > p.capacity) record_error(p.ws.hdr, DWS_ERR_CAPACITY, sum);
    }
}

// Blocks of kMergeEntries consecutive entries of one rank (blockIdx.y = rank).
__global__ void __launch_bounds__(kMergeThreads) merge_copy_kernel(MergeParams p) {
    __shared__ int s_t[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.ws.num_tensors;
    const int r = blockIdx.y;
    const long long *ro = p.rank_offsets + static_cast<long long>(r) * (T + 1);
    const long long base = static_cast<long long>(blockIdx.x) * kMergeEntries;
    if (!ws_matches(p.ws)) return;  // the offsets pass did nothing either
    if (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) != 0u) return;
    const long long n = ro[T];  // validated <= stride
    if (base >= n) return;      // uniform
    const long long last = (base + kMergeEntries < n ? base + kMergeEntries : n) - 1;
    if (warp < 2) {
        const int t = warp_tensor_of_entry(ro, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    __syncthreads();
    const int t0 = s_t[0], t1 = s_t[1];
    const long long *src_i = p.rank_indices + static_cast<long long>(r) * p.stride;
    const uint16_t *src_v = p.rank_values + static_cast<long long>(r) * p.stride;
    int tc = -1;          // tensor of the cached destination base
    long long dbase = 0;  // offsets[tc] + predecessors' entries of tc - ro[tc]
#pragma unroll 2
    for (int q = 0; q < kMergePerThread; ++q) {
        const long long j = base + tid + q * kMergeThreads;
        if (j > last) break;
        const int t = (t0 == t1) ? t0 : tensor_of_entry(ro, t0, t1, j);
        if (t != tc) {
            long long b = p.offsets[t] - ro[t];
            for (int rr = 0; rr < r; ++rr) {
                const long long *o2 = p.rank_offsets + static_cast<long long>(rr) * (T + 1);
                b += o2[t + 1] - o2[t];
            }
            tc = t;
            dbase = b;
        }
        const long long d = dbase + j;
        if (d < p.capacity) {
            p.indices[d] = __ldg(src_i + j);
            p.values[d] = __ldg(src_v + j);
        }
    }
}

}  // namespace

cudaError_t launch_merge_shards(const WsView &ws, int R, const long long *rank_offsets,
                                const long long *rank_indices, const uint16_t *rank_values,
                                long long stride, long long *offsets, long long *indices,
                                uint16_t *values, long long capacity, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = launch_delta_flag_clear(ws, s);
    if (e != cudaSuccess) return e;
    MergeParams p;
    p.ws = ws;
    p.R = R;
    p.rank_offsets = rank_offsets;
    p.rank_indices = rank_indices;
    p.rank_values = rank_values;
    p.stride = stride;
    p.offsets = offsets;
    p.indices = indices;
    p.values = values;
    p.capacity = capacity;
    long long ob = (static_cast<long long>(ws.num_tensors) + kMergeThreads) / kMergeThreads;
    if (ob > 4LL * di.sm_count) ob = 4LL * di.sm_count;
    merge_offsets_kernel<<<static_cast<unsigned int>(ob), kMergeThreads, 0, s>>>(p);
    e = launched();
    if (e != cudaSuccess || stride <= 0) return e;
    const long long bx = (stride + kMergeEntries - 1) / kMergeEntries;
    if (bx > 0x7fffffffLL || R > 65535) return cudaErrorInvalidValue;
    merge_copy_kernel<<<dim3(static_cast<unsigned int>(bx), static_cast<unsigned int>(R)),
                        kMergeThreads, 0, s>>>(p);
    return launched();
}

}  // namespace dws
