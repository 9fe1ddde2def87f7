/*
 * oracle.c -- plain, slow, single-threaded CPU reference for the delta weight
 * sync hot path.  TEST INFRASTRUCTURE ONLY (see oracle.h): only the tests,
 * the smoke check and the benchmark's CPU-baseline leg may call it.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared oracle.c -lm
 * (-ffp-contract=off keeps every float operation separately rounded, which the
 * update-model check relies on.)
 *
 * Each function is the plain definition, written out with no blocking,
 * fusion or reordering.
 */
#include "oracle.h"

#include <math.h>
#include <string.h>

/* [verl] sparse_gather.py, shard_delta_indices: compare the integer views of
 * the two snapshots, take the positions where they differ in ascending
 * order, gather the new values there.  [TRL] §4.1: the delta holds, per
 * changed parameter, those int32 indices and the bf16 values.  Here all
 * tensors share one index/value buffer and offsets[] delimits each tensor's
 * segment; a tensor with no change has an empty segment. */
int64_t ref_encode(int32_t T, const int64_t *numels,
                   const uint16_t *const *old_t, const uint16_t *const *new_t,
                   int64_t *offsets, int32_t *indices, uint16_t *values,
                   int64_t capacity)
{
    if (T < 0) return -1;
    for (int32_t t = 0; t < T; ++t)
        if (numels[t] < 0 || numels[t] > (int64_t)INT32_MAX) return -1;

    int64_t n = 0;
    offsets[0] = 0;
    for (int32_t t = 0; t < T; ++t) {
        const uint16_t *a = old_t[t];
        const uint16_t *b = new_t[t];
        for (int64_t i = 0; i < numels[t]; ++i) {
            if (a[i] != b[i]) {
                if (n < capacity) {
                    indices[n] = (int32_t)i;
                    values[n] = b[i];
                }
                ++n;
            }
        }
        offsets[t + 1] = n;
    }
    return n;
}

/* [TRL] §4.3 receive_weights: for each changed parameter,
 * snap.flatten()[indices] = values. */
int32_t ref_apply(int32_t T, const int64_t *numels, uint16_t *const *snap_t,
                  const int64_t *offsets, const int32_t *indices,
                  const uint16_t *values)
{
    if (offsets[0] != 0) return -1;
    for (int32_t t = 0; t < T; ++t) {
        if (offsets[t + 1] < offsets[t]) return -1;
        for (int64_t j = offsets[t]; j < offsets[t + 1]; ++j) {
            int64_t i = indices[j];
            if (i < 0 || i >= numels[t]) return -1;
            snap_t[t][i] = values[j];
        }
    }
    return 0;
}

/* [TRL] §4.1: a new replica takes the latest anchor and replays the deltas
 * written after it, in order. */
int32_t ref_apply_chain(int32_t T, const int64_t *numels, uint16_t *const *snap_t,
                        int32_t K, const int64_t *const *offsets_k,
                        const int32_t *const *indices_k,
                        const uint16_t *const *values_k)
{
    for (int32_t k = 0; k < K; ++k) {
        int32_t rc = ref_apply(T, numels, snap_t, offsets_k[k], indices_k[k],
                               values_k[k]);
        if (rc != 0) return rc;
    }
    return 0;
}

/* [XOR] first paragraph: the trainer XORs old and new weights bit by bit into
 * a mask of the model's size. */
void ref_xor_encode(const uint8_t *old_b, const uint8_t *new_b, uint8_t *mask,
                    int64_t nbytes)
{
    for (int64_t i = 0; i < nbytes; ++i) mask[i] = (uint8_t)(old_b[i] ^ new_b[i]);
}

/* [XOR] first paragraph: the sampler XORs the same mask into its old weights
 * and obtains the new ones, with no floating-point arithmetic. */
void ref_xor_apply(uint8_t *buf, const uint8_t *mask, int64_t nbytes)
{
    for (int64_t i = 0; i < nbytes; ++i) buf[i] = (uint8_t)(buf[i] ^ mask[i]);
}

/* The sparse form of the XOR delta at byte granularity: for each layer t and
 * byte i ascending, where old and new differ, the position i and the new
 * byte ([XOR] first paragraph: the mask is nonzero exactly there, so a
 * receiver that knows the positions and new bytes rebuilds new from old).
 * Same layout as ref_encode, positions int32.  Returns the total count, or
 * -1 on a size that does not fit int32 positions. */
int64_t ref_xor_byte_delta(int32_t T, const int64_t *nbytes,
                           const uint8_t *const *old_t, const uint8_t *const *new_t,
                           int64_t *offsets, int32_t *positions, uint8_t *values,
                           int64_t capacity)
{
    if (T < 0) return -1;
    for (int32_t t = 0; t < T; ++t)
        if (nbytes[t] < 0 || nbytes[t] > (int64_t)INT32_MAX) return -1;
    int64_t n = 0;
    offsets[0] = 0;
    for (int32_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < nbytes[t]; ++i) {
            if (old_t[t][i] != new_t[t][i]) {
                if (n < capacity) {
                    positions[n] = (int32_t)i;
                    values[n] = new_t[t][i];
                }
                ++n;
            }
        }
        offsets[t + 1] = n;
    }
    return n;
}

/* Its receiver: buf_t[positions[j]] = values[j] for each layer's segment.
 * Returns 0, or -1 at the first position outside the layer. */
int32_t ref_apply_bytes(int32_t T, const int64_t *nbytes, uint8_t *const *buf_t,
                        const int64_t *offsets, const int32_t *positions,
                        const uint8_t *values)
{
    if (offsets[0] != 0) return -1;
    for (int32_t t = 0; t < T; ++t) {
        if (offsets[t + 1] < offsets[t]) return -1;
        for (int64_t j = offsets[t]; j < offsets[t + 1]; ++j) {
            int64_t i = positions[j];
            if (i < 0 || i >= nbytes[t]) return -1;
            buf_t[t][i] = values[j];
        }
    }
    return 0;
}

uint16_t ref_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)          /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;           /* ties go to the even half */
    u += 0x7FFFu + keep_lsb;
    return (uint16_t)(u >> 16);
}

float ref_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

void ref_update_step(const uint16_t *w, const float *u, float lr, uint16_t *out,
                     int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        float wf = ref_bf16_to_float(w[i]);
        float step = lr * u[i];          /* rounded to fp32 */
        float x = wf - step;             /* rounded to fp32 */
        out[i] = ref_bf16_rne(x);
    }
}

/* [TRL] §2: bf16 keeps 7 explicit mantissa bits, so between two powers of
 * two there are 128 values and the spacing near w is about |w|*2^-7; an
 * update smaller than half that spacing is rounded away.  The exact form used
 * here: the cast leaves w's bits alone iff x lies inside w's rounding
 * interval.  The interval is bounded by the midpoints to the neighbouring
 * bf16 values below and above |w|; at an exact power of two the neighbour
 * towards zero is half as far away as the one away from zero. */
int32_t ref_absorption_changed(uint16_t w, float x)
{
    const uint16_t mag = (uint16_t)(w & 0x7FFFu);
    const int w_neg = (w >> 15) & 1;
    if (mag >= 0x7F80u) return -1;               /* w is inf or NaN */
    if (isnan(x)) return 1;                      /* cast gives NaN != finite w */

    const int x_neg = signbit(x) ? 1 : 0;
    if (x_neg != w_neg) return 1;                /* the sign bit itself changes */

    const double ax = fabs((double)x);
    const double a = fabs((double)ref_bf16_to_float(w));
    const int even = (mag & 1u) == 0;

    if (mag == 0) {
        /* ±0: the nearest non-zero bf16 is the smallest subnormal 2^-133;
         * the midpoint 2^-134 is a tie that goes to the even pattern 0. */
        return (ax <= ldexp(1.0, -134)) ? 0 : 1;
    }

    double gap_up, gap_down;
    if (mag < 0x0080u) {                         /* subnormal: fixed spacing */
        gap_up = gap_down = ldexp(1.0, -133);
    } else {
        const int e = (int)(mag >> 7) - 127;     /* |w| in [2^e, 2^(e+1)) */
        gap_up = ldexp(1.0, e - 7);
        gap_down = ((mag & 0x7Fu) == 0 && mag != 0x0080u) ? ldexp(1.0, e - 8)
                                                          : ldexp(1.0, e - 7);
    }
    const double m_lo = a - 0.5 * gap_down;
    const double m_hi = a + 0.5 * gap_up;

    if (ax > m_lo && ax < m_hi) return 0;
    if ((ax == m_lo || ax == m_hi) && even) return 0;
    return 1;
}

int64_t ref_absorption_predict(const uint16_t *w, const float *u, float lr,
                               uint8_t *changed, int64_t n)
{
    int64_t count = 0;
    for (int64_t i = 0; i < n; ++i) {
        float wf = ref_bf16_to_float(w[i]);
        float step = lr * u[i];
        float x = wf - step;
        int32_t c = ref_absorption_changed(w[i], x);
        if (c < 0) return -1;
        changed[i] = (uint8_t)c;
        count += c;
    }
    return count;
}

/* ------------------------------------------------------------------------
 * Wire positions and checksum ([verl] review, key source snippets,
 * encode.py: DeltaParam pos_start / pos_end / pos_width, checksum()).
 * ------------------------------------------------------------------------ */

int64_t ref_pack_positions(int32_t T, const int64_t *numels, const int64_t *offsets,
                           const int32_t *indices, uint8_t *positions,
                           int64_t *pos_offsets)
{
    int64_t at = 0;
    for (int32_t t = 0; t < T; ++t) {
        if (numels[t] < 0 || offsets[t + 1] < offsets[t]) return -1;
        const int width = (numels[t] <= 65536) ? 2 : 4;
        pos_offsets[t] = at;
        for (int64_t j = offsets[t]; j < offsets[t + 1]; ++j) {
            const uint32_t x = (uint32_t)indices[j];
            for (int b = 0; b < width; ++b) positions[at + b] = (uint8_t)(x >> (8 * b));
            at += width;
        }
    }
    pos_offsets[T] = at;
    return at;
}

uint64_t ref_bf16_to_f64_bits(uint16_t b)
{
    const uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    const double d = (double)f;
    uint64_t u;
    memcpy(&u, &d, sizeof u);
    return u;
}

uint64_t ref_hash_bytes(const uint8_t *b, int64_t n)
{
    uint64_t h = 0;
    for (int64_t i = 0; i < n; ++i) h ^= (uint64_t)b[i];
    return h;
}

uint64_t ref_hash_bf16(const uint16_t *v, int64_t n)
{
    uint64_t h = 0;
    for (int64_t i = 0; i < n; ++i) h ^= ref_bf16_to_f64_bits(v[i]);
    return h;
}
