// wire.cu -- the wire form of a delta: per-parameter position widths and the
// integrity checksum ([verl] review of PR #6974, key source snippets,
// encode.py: DeltaParam pos_start / pos_end / pos_width, DeltaFlush
// positions and values, checksum()).
//
// dws_pack_positions: the positions of a delta as one byte block, parameter
//   by parameter in plan order, each position in pos_width bytes
//   little-endian.  pos_width is 2 for a parameter of at most 65536 elements
//   (every position fits in 16 bits) and 4 otherwise.  A one-CTA pass scans
//   the per-parameter byte counts into pos_offsets; then every block of 2048
//   entries finds its parameters (warp-cooperative search over the delta's
//   offsets) and stores each position whole (4 bytes) where its address is
//   4-byte aligned, else as 2-byte halves.
//
// dws_checksum: hash(positions) and hash(values), where hash() XOR-reduces
//   the elements widened to 64 bits: a byte zero-extended, a bf16 value
//   converted to the IEEE double equal to it and read as a uint64 (NaNs
//   quieted with their sign and payload kept).  One grid-stride pass with
//   16-byte loads; each CTA XORs its result into the outputs once.  The
//   checksum of the pages is hash(positions) ^ (hash(values) << 1) on
//   unbounded integers, a 65-bit number: a one-thread kernel after the hashes
//   writes it as a 128-bit little-endian integer (two uint64 words, bit 64 the
//   only bit of the high word that can be set).
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr long long kSmallTensor = 65536;  // at most this many elements: 2-byte positions
constexpr int kPackThreads = 256;
constexpr int kPackPerThread = 8;
constexpr int kPackEntries = kPackThreads * kPackPerThread;
constexpr int kScanThreads = 1024;

__device__ __forceinline__ int pos_width_of(long long numel) { return numel <= kSmallTensor ? 2 : 4; }

// pos_offsets[t] = sum over t' < t of width(t') * (offsets[t'+1] - offsets[t']);
// pos_offsets[T] = the block's size.  One CTA, chunks of kScanThreads tensors.
__global__ void __launch_bounds__(kScanThreads) pos_offsets_kernel(WsView ws, const long long *offsets,
                                                                   long long *pos_offsets,
                                                                   long long pos_capacity) {
    __shared__ long long warp_sums[kScanThreads / 32];
    __shared__ long long carry;
    if (!ws_matches(ws)) return;
    if (ld_relaxed_gpu_u32(&ws.hdr->delta_bad) != 0u) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = ws.num_tensors;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < T; base += kScanThreads) {
        const int t = base + tid;
        long long v = 0;
        if (t < T) v = pos_width_of(ws.numel[t]) * (offsets[t + 1] - offsets[t]);
        long long incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long u = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += u;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        long long before = carry;
        for (int w = 0; w < warp; ++w) before += warp_sums[w];
        if (t < T) pos_offsets[t] = before + incl - v;
        __syncthreads();
        if (tid == kScanThreads - 1) carry = before + incl;
        __syncthreads();
    }
    if (tid == 0) {
        pos_offsets[T] = carry;
        if (carry > pos_capacity) record_error(ws.hdr, DWS_ERR_CAPACITY, carry);
    }
}

struct PackParams {
    WsView ws;
    DeltaRef d;
    const long long *pos_offsets;
    uint8_t *positions;
    long long pos_capacity;
};

__global__ void __launch_bounds__(kPackThreads) pack_positions_kernel(PackParams p) {
    __shared__ int s_t[2];
    __shared__ int s_go;
    __shared__ long long s_end;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.ws.num_tensors;
    const long long base = static_cast<long long>(blockIdx.x) * kPackEntries;
    const long long cap = p.d.count;
    if (base >= cap) return;  // uniform
    int idx[kPackPerThread];
#pragma unroll
    for (int r = 0; r < kPackPerThread; ++r) {
        const long long j = base + tid + r * kPackThreads;
        if (j < cap) idx[r] = __ldg(p.d.indices + j);
    }
    if (warp < 2) {
        const long long last = (base + kPackEntries < cap ? base + kPackEntries : cap) - 1;
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
        s_end = (base + kPackEntries < total) ? base + kPackEntries : total;
        s_go = ok && (ld_relaxed_gpu_u32(&p.ws.hdr->delta_bad) == 0u) && base < s_end;
    }
    __syncthreads();
    if (!s_go) return;
    const long long end = s_end;
    const int t0 = s_t[0], t1 = s_t[1];
    // the block's first tensor, read once (a block inside one tensor, the
    // common case, needs nothing else)
    const long long n0 = p.ws.numel[t0], pb0 = p.pos_offsets[t0], ob0 = p.d.offsets[t0];
    if (t0 == t1 && pos_width_of(n0) == 4) {
        // 4-byte positions of one tensor: the block's positions are its
        // indices, stored contiguously from at0 (checked once for room)
        const long long at0 = pb0 + (base - ob0) * 4;
        uint8_t *dst0 = p.positions + at0;
        if (at0 >= 0 && at0 + (end - base) * 4 <= p.pos_capacity && (reinterpret_cast<uintptr_t>(dst0) & 3u) == 0) {
            uint32_t *d32 = reinterpret_cast<uint32_t *>(dst0);
            const int m = static_cast<int>(end - base);
            long long bad_j = -1;
#pragma unroll
            for (int r = 0; r < kPackPerThread; ++r) {
                const int q = tid + r * kPackThreads;
                if (q < m) {
                    if (static_cast<unsigned long long>(static_cast<long long>(idx[r])) < static_cast<unsigned long long>(n0))
                        d32[q] = static_cast<uint32_t>(idx[r]);
                    else if (bad_j < 0)
                        bad_j = base + q;
                }
            }
            if (bad_j >= 0) record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, bad_j);
            return;
        }
    }
#pragma unroll
    for (int r = 0; r < kPackPerThread; ++r) {
        const long long j = base + tid + r * kPackThreads;
        if (j >= end) continue;
        int t = t0;
        long long n = n0, pb = pb0, ob = ob0;
        if (t0 != t1) {
            t = tensor_of_entry(p.d.offsets, t0, t1, j);
            n = p.ws.numel[t];
            pb = p.pos_offsets[t];
            ob = p.d.offsets[t];
        }
        const int i = idx[r];
        if (i < 0 || static_cast<long long>(i) >= n) {
            record_error(p.ws.hdr, DWS_ERR_BAD_DELTA, j);
            continue;
        }
        const int w = pos_width_of(n);
        const long long at = pb + (j - ob) * w;
        if (at + w > p.pos_capacity) continue;  // recorded by the offsets pass
        uint8_t *dst = p.positions + at;  // even
        if (w == 4 && (reinterpret_cast<uintptr_t>(dst) & 3u) == 0) {
            *reinterpret_cast<uint32_t *>(dst) = static_cast<uint32_t>(i);
        } else {
            uint16_t *d16 = reinterpret_cast<uint16_t *>(dst);
            d16[0] = static_cast<uint16_t>(i & 0xffff);
            if (w == 4) d16[1] = static_cast<uint16_t>(static_cast<uint32_t>(i) >> 16);
        }
    }
}

constexpr int kSumThreads = 512;

__device__ __forceinline__ unsigned long long fold_bytes(unsigned long long x) {
    x ^= x >> 32;
    x ^= x >> 16;
    x ^= x >> 8;
    return x & 0xffull;
}

__global__ void __launch_bounds__(kSumThreads) checksum_kernel(const uint8_t *pos, long long nbytes,
                                                               const uint16_t *val, long long nval,
                                                               unsigned long long *out) {
    const long long stride = static_cast<long long>(gridDim.x) * kSumThreads;
    const long long gid = static_cast<long long>(blockIdx.x) * kSumThreads + threadIdx.x;
    unsigned long long hp = 0, hv = 0;
    // bytes: unaligned head and tail one by one, the middle as 16-byte words
    const uintptr_t pa = reinterpret_cast<uintptr_t>(pos);
    long long head = static_cast<long long>((16 - (pa & 15u)) & 15u);
    if (head > nbytes) head = nbytes;
    const long long nvec = (nbytes - head) >> 4;
    if (gid < head) hp ^= pos[gid];
    const uint4 *pv = reinterpret_cast<const uint4 *>(pos + head);
    unsigned long long words = 0;
    for (long long k = gid; k < nvec; k += 4 * stride) {  // four loads in flight
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            w[u] = k + u * stride < nvec ? ld_stream_v4(pv + k + u * stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            words ^= (static_cast<unsigned long long>(w[u].y) << 32 | w[u].x) ^
                     (static_cast<unsigned long long>(w[u].w) << 32 | w[u].z);
    }
    hp ^= fold_bytes(words);
    for (long long k = head + (nvec << 4) + gid; k < nbytes; k += stride) hp ^= pos[k];
    // values: unaligned head, 8 per 16-byte word, tail
    const uintptr_t va = reinterpret_cast<uintptr_t>(val);
    long long vhead = ((va & 15u) == 0) ? 0 : static_cast<long long>((16 - (va & 15u)) >> 1);
    if ((va & 1u) != 0u || vhead > nval) vhead = nval;  // odd address: all one by one
    const long long vvec = (nval - vhead) >> 3;
    if (gid < vhead) hv ^= bf16_to_f64_bits(val[gid]);
    const uint4 *vv = reinterpret_cast<const uint4 *>(val + vhead);
    // A normal bf16 (exponent 1..254) is the double with bits sign << 63 |
    // (e + 896) << 52 | m << 45: three disjoint fields, so their XORs over many
    // values can be kept apart and assembled once.  sm2 folds sign and
    // mantissa bits two values at a time (one 32-bit word); ex folds e + 896.
    // Zeros, subnormals, infinities and NaNs take the exact conversion.
    uint32_t sm2 = 0u, ex = 0u;
    for (long long k = gid; k < vvec; k += 4 * stride) {  // four loads in flight
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = k + u * stride < vvec ? ld_stream_v4(vv + k + u * stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // a zero word past the end is +0.0: double bits 0
            const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t el = (ws[q] >> 7) & 0xffu, eh = (ws[q] >> 23) & 0xffu;
                if (el - 1u < 254u && eh - 1u < 254u) {
                    sm2 ^= ws[q] & 0x807f807fu;
                    ex ^= (el + 896u) ^ (eh + 896u);
                } else {
                    hv ^= bf16_to_f64_bits(ws[q] & 0xffffu) ^ bf16_to_f64_bits(ws[q] >> 16);
                }
            }
        }
    }
    {
        const uint32_t sgn = ((sm2 >> 15) ^ (sm2 >> 31)) & 1u;
        const uint32_t man = (sm2 ^ (sm2 >> 16)) & 0x7fu;
        hv ^= (static_cast<unsigned long long>(sgn) << 63) | (static_cast<unsigned long long>(ex & 0x7ffu) << 52) |
              (static_cast<unsigned long long>(man) << 45);
    }
    for (long long k = vhead + (vvec << 3) + gid; k < nval; k += stride) hv ^= bf16_to_f64_bits(val[k]);
    // CTA reduction, one atomic per output per CTA
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        hp ^= __shfl_xor_sync(0xffffffffu, hp, d);
        hv ^= __shfl_xor_sync(0xffffffffu, hv, d);
    }
    __shared__ unsigned long long sp[kSumThreads / 32], sv[kSumThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sp[warp] = hp;
        sv[warp] = hv;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long a = 0, b = 0;
        for (int w = 0; w < kSumThreads / 32; ++w) {
            a ^= sp[w];
            b ^= sv[w];
        }
        if (a) atomicXor(out, a);
        if (b) atomicXor(out + 1, b);
    }
}

// checksum = hash(positions) ^ (hash(values) << 1), the shift taken on a
// 128-bit integer so that bit 63 of hash(values) lands in bit 64.
__global__ void checksum_wire_kernel(const unsigned long long *hashes, unsigned long long *wire) {
    if (threadIdx.x != 0) return;
    const unsigned long long hp = hashes[0], hv = hashes[1];
    wire[0] = hp ^ (hv << 1);
    wire[1] = hv >> 63;
}

}  // namespace

cudaError_t launch_checksum_wire(const unsigned long long *hashes, unsigned long long *wire,
                                 cudaStream_t s) {
    checksum_wire_kernel<<<1, 32, 0, s>>>(hashes, wire);
    return launched();
}

cudaError_t launch_pack_positions(const WsView &ws, const DeltaRef &d, uint8_t *positions,
                                  long long pos_capacity, long long *pos_offsets, cudaStream_t s) {
    cudaError_t e = launch_delta_check(ws, &d, 1, s);
    if (e != cudaSuccess) return e;
    pos_offsets_kernel<<<1, kScanThreads, 0, s>>>(ws, d.offsets, pos_offsets, pos_capacity);
    e = launched();
    if (e != cudaSuccess) return e;
    if (d.count <= 0) return cudaSuccess;
    PackParams p;
    p.ws = ws;
    p.d = d;
    p.pos_offsets = pos_offsets;
    p.positions = positions;
    p.pos_capacity = pos_capacity;
    const long long blocks = (d.count + kPackEntries - 1) / kPackEntries;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    pack_positions_kernel<<<static_cast<unsigned int>(blocks), kPackThreads, 0, s>>>(p);
    return launched();
}

cudaError_t launch_checksum(const uint8_t *positions, long long nbytes, const uint16_t *values,
                            long long nval, unsigned long long *out, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(out, 0, 2 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    const long long work = (nbytes >> 4) + (nval >> 3) + 1;
    long long grid = (work + kSumThreads - 1) / kSumThreads;
    const long long cap = 4LL * di.sm_count;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    checksum_kernel<<<static_cast<unsigned int>(grid), kSumThreads, 0, s>>>(positions, nbytes, values,
                                                                            nval, out);
    return launched();
}

}  // namespace dws
