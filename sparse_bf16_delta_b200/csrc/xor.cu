// xor.cu -- the XOR-mask variant (humans& weight-sync summary, paragraph 1:
// mask = old ^ new bit by bit, the same size as the model; the receiver gets
// new = old ^ mask with no floating-point arithmetic).
//
// out[b] = a[b] ^ c[b].  Encode: a = old, c = new, out = mask.  Apply:
// a = out = buf, c = mask (in place).
//
// A pure HBM stream (2 bytes read + 1 written per byte of model).  When the
// three pointers share their alignment modulo 16, the body moves in 16-byte
// vectors, four per thread per iteration with all loads issued before the
// XORs (8 x 16 B in flight per thread), read-once data bypassing L1 and
// stores marked streaming; the unaligned head and the tail go byte by byte.
// Pointers with different alignments take a plain byte loop.
#include <cuda_runtime.h>

#include "dws_internal.cuh"

namespace dws {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) xor_vec_kernel(const uint8_t *a, const uint8_t *c,
                                                           uint8_t *out, long long head,
                                                           long long nvec, long long nbytes) {
    const long long tid = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x;
    const long long nthreads = static_cast<long long>(gridDim.x) * kThreads;
    const uint4 *av = reinterpret_cast<const uint4 *>(a + head);
    const uint4 *cv = reinterpret_cast<const uint4 *>(c + head);
    uint4 *ov = reinterpret_cast<uint4 *>(out + head);
    const bool in_place = (a == out);

    long long v = tid;
    for (; v + (kUnroll - 1) * nthreads < nvec; v += kUnroll * nthreads) {
        uint4 x[kUnroll], y[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long k = v + u * nthreads;
            x[u] = in_place ? av[k] : ld_stream_v4(av + k);
            y[u] = ld_stream_v4(cv + k);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint4 r = make_uint4(x[u].x ^ y[u].x, x[u].y ^ y[u].y, x[u].z ^ y[u].z,
                                       x[u].w ^ y[u].w);
            st_stream_v4(ov + v + u * nthreads, r);
        }
    }
    for (; v < nvec; v += nthreads) {
        const uint4 x = in_place ? av[v] : ld_stream_v4(av + v);
        const uint4 y = ld_stream_v4(cv + v);
        st_stream_v4(ov + v, make_uint4(x.x ^ y.x, x.y ^ y.y, x.z ^ y.z, x.w ^ y.w));
    }
    // Unaligned head [0, head) and tail [head + 16*nvec, nbytes).
    const long long tail0 = head + 16 * nvec;
    const long long extra = head + (nbytes - tail0);
    for (long long i = tid; i < extra; i += nthreads) {
        const long long b = (i < head) ? i : tail0 + (i - head);
        out[b] = static_cast<uint8_t>(a[b] ^ c[b]);
    }
}

__global__ void __launch_bounds__(kThreads) xor_byte_kernel(const uint8_t *a, const uint8_t *c,
                                                            uint8_t *out, long long nbytes) {
    const long long nthreads = static_cast<long long>(gridDim.x) * kThreads;
    for (long long i = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; i < nbytes;
         i += nthreads) {
        out[i] = static_cast<uint8_t>(a[i] ^ c[i]);
    }
}

}  // namespace

cudaError_t launch_xor(const uint8_t *a, const uint8_t *c, uint8_t *out, long long nbytes,
                       cudaStream_t s) {
    if (nbytes <= 0) return cudaSuccess;
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    const uintptr_t ma = reinterpret_cast<uintptr_t>(a) & 15u;
    const uintptr_t mc = reinterpret_cast<uintptr_t>(c) & 15u;
    const uintptr_t mo = reinterpret_cast<uintptr_t>(out) & 15u;
    long long blocks_cap = 8LL * di.sm_count;
    if (ma == mc && ma == mo) {
        long long head = static_cast<long long>((16u - ma) & 15u);
        if (head > nbytes) head = nbytes;
        const long long nvec = (nbytes - head) / 16;
        long long blocks = (nvec + kThreads * kUnroll - 1) / (kThreads * kUnroll);
        if (blocks > blocks_cap) blocks = blocks_cap;
        if (blocks < 1) blocks = 1;
        xor_vec_kernel<<<static_cast<unsigned int>(blocks), kThreads, 0, s>>>(a, c, out, head,
                                                                              nvec, nbytes);
    } else {
        long long blocks = (nbytes + kThreads - 1) / kThreads;
        if (blocks > blocks_cap) blocks = blocks_cap;
        xor_byte_kernel<<<static_cast<unsigned int>(blocks), kThreads, 0, s>>>(a, c, out, nbytes);
    }
    return launched();
}

}  // namespace dws
