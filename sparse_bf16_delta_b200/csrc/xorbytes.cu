// xorbytes.cu -- the sparse XOR delta of packed byte layers at byte
// granularity (the humans& weight-sync summary, first paragraph: the XOR mask
// of old and new is nonzero exactly at the changed bytes, so the delta can be
// shipped as their positions and new values: 4 + 1 bytes per changed byte).
//
// The layers are encoded as 16-bit words by dws_encode (one entry per changed
// word: 6 bytes); this file turns that word delta into the byte delta and
// scatters a byte delta back:
//
//   bytes_count_kernel   blocks of 2048 word entries: each entry's changed
//     bytes (1 or 2: its low byte at 2i, its high byte at 2i + 1) from the
//     old word and the entry's new word; one count per block.
//   bytes_scan_kernel    one CTA: exclusive scan of the block counts, the
//     total, and the offsets of layers with no entry at or after theirs.
//   bytes_write_kernel   the same blocks again: a block-local scan places
//     each entry's bytes after those of the entries before it; the first
//     entry of a layer writes that layer's byte offset.
//   apply_bytes_kernel   one byte delta onto byte layers, every position
//     range- and order-checked (as dws_apply).
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kBThreads = 256;
constexpr int kBPerThread = 8;
constexpr int kBEntries = kBThreads * kBPerThread;  // word entries per block
constexpr int kBScanThreads = 1024;

struct BytesParams {
    WsView ws;
    const uint16_t *const *old_ptrs;  // the old layers, as 16-bit words
    DeltaRef d;                       // the word delta
    long long limit;                  // word entries read: min(count, elements of the plan)
    long long *counts;                // per block: byte entries, then (after the scan) the block's first
    long long *byte_offsets;          // [T + 1]
    int *positions;
    uint8_t *values;
    long long capacity;
};

// Word entry j's changed-byte mask (bit 0: low byte, bit 1: high byte; 0 if
// the entry is bad) and new word.
struct WordEntry {
    unsigned int mask;
    uint32_t w;
    int i;
    int t;
};

// The entries of this thread (j = base + tid + r * kBThreads) with their
// tensor and checks.  Shared by the count and the write pass, which must see
// the same masks.  Returns false when the block has nothing to do.
__device__ __forceinline__ bool load_block(const BytesParams &p, long long base, WordEntry (&e)[kBPerThread],
                                           long long *end_out, bool record) {
    __shared__ int s_t[2];
    __shared__ int s_go;
    __shared__ long long s_end;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.ws.num_tensors;
    int idx[kBPerThread];
    uint16_t val[kBPerThread];
#pragma unroll
    for (int r = 0; r < kBPerThread; ++r) {
        const long long j = base + tid + r * kBThreads;
        idx[r] = 0;
        val[r] = 0;
        if (j < p.limit) {
            idx[r] = __ldg(p.d.indices + j);
            val[r] = __ldg(p.d.values + j);
        }
    }
    if (warp < 2) {
        const long long last = (base + kBEntries < p.limit ? base + kBEntries : p.limit) - 1;
        const int t = warp_tensor_of_entry(p.d.offsets, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    if (tid == 64) {
        const WsHeader *h = p.ws.hdr;
        const bool ok = (h->magic == kWsMagic && h->fingerprint == p.ws.fingerprint &&
                         h->num_tiles == p.ws.num_tiles && h->num_tensors == T);
        if (!ok && record) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, 0);
        const long long nnz = p.d.offsets[T];
        const long long total = nnz < p.limit ? nnz : p.limit;
        s_end = (base + kBEntries < total) ? base + kBEntries : total;
        s_go = ok && (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) == 0u);
    }
    __syncthreads();
    *end_out = s_end;
    if (!s_go) return false;
    const int t0 = s_t[0], t1 = s_t[1];
#pragma unroll
    for (int r = 0; r < kBPerThread; ++r) {
        const long long j = base + tid + r * kBThreads;
        e[r].mask = 0u;
        e[r].w = 0u;
        e[r].i = 0;
        e[r].t = 0;
        int prev = __shfl_up_sync(0xffffffffu, idx[r], 1);
        if (j >= s_end) continue;
        const int t = (t0 == t1) ? t0 : tensor_of_entry(p.d.offsets, t0, t1, j);
        e[r].t = t;  // also for a bad entry: the write pass places layer offsets by it
        const long long n = p.ws.numel[t];
        const int i = idx[r];
        bool ok = i >= 0 && static_cast<long long>(i) < n;
        if (ok && j > p.d.offsets[t]) {
            if (lane == 0) prev = __ldg(p.d.indices + j - 1);
            ok = prev < i;
        }
        const uint16_t *op = p.old_ptrs[t];
        if (!ok || op == nullptr || (reinterpret_cast<uintptr_t>(op) & 1u)) {
            if (record) record_error(p.ws.hdr, ok ? DWS_ERR_INVALID : DWS_ERR_BAD_DELTA, j);
            continue;
        }
        const uint32_t x = static_cast<uint32_t>(op[i] ^ val[r]);
        e[r].mask = ((x & 0xffu) != 0u ? 1u : 0u) | ((x >> 8) != 0u ? 2u : 0u);
        e[r].w = val[r];
        e[r].i = i;
    }
    return true;
}

__global__ void __launch_bounds__(kBThreads) bytes_count_kernel(BytesParams p) {
    __shared__ int s_warp[kBThreads / 32];
    WordEntry e[kBPerThread];
    long long end;
    const long long base = static_cast<long long>(blockIdx.x) * kBEntries;
    const bool go = load_block(p, base, e, &end, true);
    int c = 0;
    if (go) {
#pragma unroll
        for (int r = 0; r < kBPerThread; ++r) c += __popc(e[r].mask);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long sum = 0;
        for (int w = 0; w < kBThreads / 32; ++w) sum += s_warp[w];
        p.counts[blockIdx.x] = sum;
    }
}

// One CTA: counts[b] <- bytes of the blocks before b; byte_offsets[T] and
// the offsets of layers whose first word entry is at or past the end.
__global__ void __launch_bounds__(kBScanThreads) bytes_scan_kernel(BytesParams p, long long nblocks) {
    __shared__ long long s_warp[kBScanThreads / 32];
    __shared__ long long s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (long long b0 = 0; b0 < nblocks; b0 += kBScanThreads) {
        const long long b = b0 + tid;
        const long long v = b < nblocks ? p.counts[b] : 0;
        long long incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        long long before = s_carry;
        for (int w = 0; w < warp; ++w) before += s_warp[w];
        if (b < nblocks) p.counts[b] = before + incl - v;
        __syncthreads();
        if (tid == kBScanThreads - 1) s_carry = before + incl;
        __syncthreads();
    }
    const long long total = s_carry;
    const int T = p.ws.num_tensors;
    const long long nnz = p.d.offsets[T];
    // more entries than the plan has words: some word is listed twice
    if (tid == 0 && nnz > p.limit) record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, p.limit);
    for (int t = tid; t <= T; t += kBScanThreads)
        if (p.d.offsets[t] >= nnz) p.byte_offsets[t] = total;
    if (tid == 0 && total > p.capacity) record_error(p.ws.hdr, DWS_ERR_CAPACITY, total);
}

__global__ void __launch_bounds__(kBThreads) bytes_write_kernel(BytesParams p) {
    __shared__ int s_warp[kBThreads / 32];
    WordEntry e[kBPerThread];
    long long end;
    const long long base = static_cast<long long>(blockIdx.x) * kBEntries;
    const bool go = load_block(p, base, e, &end, false);
    if (!go) return;  // uniform
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Entries are taken in the order j = base + tid + r * kBThreads: the
    // byte entries of round r follow all those of rounds before it, so the
    // block's scan runs round by round.
    long long start = p.counts[blockIdx.x];
#pragma unroll
    for (int r = 0; r < kBPerThread; ++r) {
        const int c = __popc(e[r].mask);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        int before = 0, round = 0;
#pragma unroll
        for (int w = 0; w < kBThreads / 32; ++w) {
            const int v = s_warp[w];
            before += w < warp ? v : 0;
            round += v;
        }
        __syncthreads();  // s_warp is reused by the next round
        const long long at = start + before + incl - c;
        const long long j = base + tid + r * kBThreads;
        if (j < end) {
            const int t = e[r].t;
            if (j == p.d.offsets[t]) {
                // the layer's first word entry: its byte offset, and that
                // of the empty layers just before it
                p.byte_offsets[t] = at;
                for (int u = t - 1; u >= 0 && p.d.offsets[u] == j; --u) p.byte_offsets[u] = at;
            }
            long long k = at;
            if ((e[r].mask & 1u) && k < p.capacity) {
                p.positions[k] = 2 * e[r].i;
                p.values[k] = static_cast<uint8_t>(e[r].w & 0xffu);
            }
            k += e[r].mask & 1u;
            if ((e[r].mask & 2u) && k < p.capacity) {
                p.positions[k] = 2 * e[r].i + 1;
                p.values[k] = static_cast<uint8_t>(e[r].w >> 8);
            }
        }
        start += round;
    }
}

// ---------------------------------------------------------------------------
// Apply of a byte delta
// ---------------------------------------------------------------------------
struct ApplyBytesParams {
    WsView ws;
    uint8_t *const *buf_ptrs;
    const long long *offsets;
    const int *positions;
    const uint8_t *values;
    long long count;
};

__global__ void __launch_bounds__(kBThreads) apply_bytes_kernel(ApplyBytesParams p) {
    __shared__ int s_t[2];
    __shared__ int s_go;
    __shared__ long long s_end;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.ws.num_tensors;
    const long long base = static_cast<long long>(blockIdx.x) * kBEntries;
    if (base >= p.count) return;  // uniform
    int pos[kBPerThread];
    uint8_t val[kBPerThread];
#pragma unroll
    for (int r = 0; r < kBPerThread; ++r) {
        const long long j = base + tid + r * kBThreads;
        pos[r] = 0;
        val[r] = 0;
        if (j < p.count) {
            pos[r] = __ldg(p.positions + j);
            val[r] = __ldg(p.values + j);
        }
    }
    if (warp < 2) {
        const long long last = (base + kBEntries < p.count ? base + kBEntries : p.count) - 1;
        const int t = warp_tensor_of_entry(p.offsets, T, warp == 0 ? base : last);
        if (lane == 0) s_t[warp] = t;
    }
    if (tid == 64) {
        const WsHeader *h = p.ws.hdr;
        const bool ok = (h->magic == kWsMagic && h->fingerprint == p.ws.fingerprint &&
                         h->num_tiles == p.ws.num_tiles && h->num_tensors == T);
        if (!ok) record_error(p.ws.hdr, DWS_ERR_WORKSPACE, 0);
        const long long nnz = p.offsets[T];
        const long long total = nnz < p.count ? nnz : p.count;
        s_end = (base + kBEntries < total) ? base + kBEntries : total;
        s_go = ok && (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) == 0u) && base < s_end;
    }
    __syncthreads();
    if (!s_go) return;
    const long long end = s_end;
    const int t0 = s_t[0], t1 = s_t[1];
#pragma unroll
    for (int r = 0; r < kBPerThread; ++r) {
        const long long j = base + tid + r * kBThreads;
        int prev = __shfl_up_sync(0xffffffffu, pos[r], 1);
        if (j >= end) continue;
        const int t = (t0 == t1) ? t0 : tensor_of_entry(p.offsets, t0, t1, j);
        const long long nbytes = 2 * p.ws.numel[t];
        const int i = pos[r];
        bool ok = i >= 0 && static_cast<long long>(i) < nbytes;
        if (ok && j > p.offsets[t]) {
            if (lane == 0) prev = __ldg(p.positions + j - 1);
            ok = prev < i;
        }
        uint8_t *dst = p.buf_ptrs[t];
        if (ok && dst != nullptr) {
            dst[i] = val[r];
        } else {
            record_error(p.ws.hdr, ok ? DWS_ERR_INVALID : DWS_ERR_BAD_DELTA, j);
        }
    }
}

}  // namespace

cudaError_t launch_xor_bytes_from_words(const WsView &ws, const uint16_t *const *old_ptrs, const DeltaRef &d,
                                        long long plan_elems, long long *byte_offsets, int *positions,
                                        uint8_t *values, long long capacity, cudaStream_t s) {
    cudaError_t e = launch_delta_check(ws, &d, 1, s);
    if (e != cudaSuccess) return e;
    BytesParams p;
    p.ws = ws;
    p.old_ptrs = old_ptrs;
    p.d = d;
    p.limit = d.count < plan_elems ? d.count : plan_elems;  // a valid delta has at most one entry per word
    p.counts = reinterpret_cast<long long *>(ws.tile_status);
    p.byte_offsets = byte_offsets;
    p.positions = positions;
    p.values = values;
    p.capacity = capacity;
    const long long nb = (p.limit + kBEntries - 1) / kBEntries;
    // the block counts live in the per-call scratch: 32 bytes per tile
    if (nb > 4 * ws.num_tiles || nb > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (nb > 0) {
        bytes_count_kernel<<<static_cast<unsigned int>(nb), kBThreads, 0, s>>>(p);
        e = launched();
        if (e != cudaSuccess) return e;
    }
    bytes_scan_kernel<<<1, kBScanThreads, 0, s>>>(p, nb);
    e = launched();
    if (e != cudaSuccess) return e;
    if (nb > 0) {
        bytes_write_kernel<<<static_cast<unsigned int>(nb), kBThreads, 0, s>>>(p);
        e = launched();
    }
    return e;
}

cudaError_t launch_apply_bytes(const WsView &ws, uint8_t *const *buf_ptrs, const long long *offsets,
                               const int *positions, const uint8_t *values, long long count, cudaStream_t s) {
    DeltaRef d{offsets, positions, nullptr, count};
    cudaError_t e = launch_delta_check(ws, &d, 1, s);
    if (e != cudaSuccess) return e;
    if (count <= 0) return cudaSuccess;
    ApplyBytesParams p;
    p.ws = ws;
    p.buf_ptrs = buf_ptrs;
    p.offsets = offsets;
    p.positions = positions;
    p.values = values;
    p.count = count;
    const long long blocks = (count + kBEntries - 1) / kBEntries;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    apply_bytes_kernel<<<static_cast<unsigned int>(blocks), kBThreads, 0, s>>>(p);
    return launched();
}

}  // namespace dws
