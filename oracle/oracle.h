/*
 * oracle.h -- plain, slow, single-threaded CPU reference for the delta weight
 * sync hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this code: it exists so that the tests, the smoke check and the
 * benchmark's CPU-baseline leg can compare the CUDA library against an
 * implementation that a reader can check against the source pages by eye.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [TRL]   "Shipping a Trillion Parameters With a Hub Bucket: Delta Weight
 *           Sync in TRL" (Korean translation of the Hugging Face blog), and
 *           its Chinese summary "TRL 中的 Delta Weight Sync ...".
 *   [verl]  review of verl PR #6974 "delta_sharded" engine, section
 *           "关键源码片段" (key source snippets), sparse_gather.py.
 *   [XOR]   "همگام‌سازی وزن‌ها تو RL با کمتر از ۰.۲۳ ثانیه توقف" (humans&
 *           weight sync summary), first and third paragraphs.
 *
 * Every value is handled as raw bits: bf16 as uint16_t, the XOR path as
 * uint8_t.  Floating point appears only in the update-model and absorption
 * checks (ref_update_step, ref_absorption_changed, ref_bf16_rne), which pin
 * the synthetic inputs to the rounding argument of [TRL] §2.
 *
 * Error behaviour: functions that take sizes return -1 (or set nothing) on an
 * invalid size; they never abort.
 */
#ifndef DWS_ORACLE_H
#define DWS_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Sparse delta encode, [verl] sparse_gather.py shard_delta_indices and [TRL]
 * §4.1 (per changed parameter: int32 element indices + bf16 values).
 * For t = 0..T-1 in table order and i = 0..numels[t]-1 ascending, an element
 * is "changed" iff its 16-bit pattern differs between old and new; its local
 * index i and the new bits are appended.  offsets[t] .. offsets[t+1] is the
 * segment of tensor t (offsets has T+1 entries, offsets[0] = 0).
 * Entries beyond `capacity` are counted but not stored.
 * Returns the total number of changed elements, or -1 if some numel is
 * negative or >= 2^31 (indices are int32). */
int64_t ref_encode(int32_t T, const int64_t *numels,
                   const uint16_t *const *old_t, const uint16_t *const *new_t,
                   int64_t *offsets, int32_t *indices, uint16_t *values,
                   int64_t capacity);

/* Receiver-side scatter, [TRL] §4.3 (snap.flatten()[indices] = values):
 * for each tensor t and j in [offsets[t], offsets[t+1]):
 *   snap_t[indices[j]] = values[j].
 * Returns 0, or -1 (and stops) at the first entry whose index is outside
 * [0, numels[t]) or whose offsets are not monotone. */
int32_t ref_apply(int32_t T, const int64_t *numels, uint16_t *const *snap_t,
                  const int64_t *offsets, const int32_t *indices,
                  const uint16_t *values);

/* Anchor + delta chain, [TRL] §4.1 (anchor every N syncs, a new replica
 * replays the deltas after the latest anchor): ref_apply for k = 0..K-1 in
 * order, so a later delta wins where two touch the same element. */
int32_t ref_apply_chain(int32_t T, const int64_t *numels, uint16_t *const *snap_t,
                        int32_t K, const int64_t *const *offsets_k,
                        const int32_t *const *indices_k,
                        const uint16_t *const *values_k);

/* XOR-mask variant, [XOR] first paragraph: mask = old ^ new (same size as
 * the model), and the receiver recovers new = old ^ mask. */
void ref_xor_encode(const uint8_t *old_b, const uint8_t *new_b, uint8_t *mask,
                    int64_t nbytes);
void ref_xor_apply(uint8_t *buf, const uint8_t *mask, int64_t nbytes);

/* fp32 -> bf16 round-to-nearest-even on the fp32 bit pattern (add 0x7FFF
 * plus the lowest kept bit, then truncate); NaN inputs stay NaN with the
 * quiet bit set. */
uint16_t ref_bf16_rne(float x);

/* bf16 bits -> float (exact: bf16 is the top half of an fp32). */
float ref_bf16_to_float(uint16_t b);

/* The synthetic optimizer step the workloads use: for each element,
 *   x = fl32( fl32(w) - fl32(lr * u) ),  out = bf16_rne(x)
 * with every operation rounded to fp32 separately (no fused multiply-add). */
void ref_update_step(const uint16_t *w, const float *u, float lr, uint16_t *out,
                     int64_t n);

/* Absorption rule, [TRL] §2: a bf16 weight w keeps its bits after the cast
 * iff the updated fp32 value x lies strictly inside the rounding interval of
 * w, i.e. between the midpoints to w's lower and upper bf16 neighbours, or
 * exactly on a midpoint when w's last mantissa bit is even (ties to even).
 * Computed with exact midpoints in double precision, independently of the
 * integer rounding in ref_bf16_rne.  Returns 1 if the bits change, 0 if the
 * update is absorbed, -1 if w is not finite. */
int32_t ref_absorption_changed(uint16_t w, float x);

/* Convenience over arrays: changed[i] = ref_absorption_changed(w[i], x_i)
 * where x_i = fl32(fl32(w[i]) - fl32(lr*u[i])).  Returns the number of
 * predicted changes, or -1 if some w is not finite. */
int64_t ref_absorption_predict(const uint16_t *w, const float *u, float lr,
                               uint8_t *changed, int64_t n);

/* Wire positions, [verl] review, key source snippets, encode.py: a flush
 * carries its positions as one uint8 byte block; each parameter's positions
 * occupy bytes [pos_start, pos_end) of it, pos_width (2 or 4) bytes each.
 * The page does not say when 2 is used; the reading taken here: 2 bytes when
 * every position of the parameter fits in 16 bits (numels[t] <= 65536), else
 * 4.  Positions are written little-endian, parameters in table order.
 * pos_offsets (T+1 entries) receives the byte starts; pos_offsets[T] = total.
 * Returns the total number of bytes, or -1 on a negative numel or
 * non-monotone offsets.  `positions` must hold the total. */
int64_t ref_pack_positions(int32_t T, const int64_t *numels, const int64_t *offsets,
                           const int32_t *indices, uint8_t *positions,
                           int64_t *pos_offsets);

/* The wire checksum, [verl] encode.py checksum(): hash(positions) XOR
 * (hash(values) << 1), where hash() XOR-reduces the elements after widening
 * each one to its 64-bit equivalent (an unsigned byte zero-extended; a bf16
 * value converted to an IEEE double) and reading that as a uint64.  The two
 * hashes are returned separately: the shift makes the checksum a 65-bit
 * number. */
uint64_t ref_hash_bytes(const uint8_t *b, int64_t n);
uint64_t ref_hash_bf16(const uint16_t *v, int64_t n);

/* The 64-bit pattern of the double equal to a bf16 value (for NaN, the C
 * conversion on this host). */
uint64_t ref_bf16_to_f64_bits(uint16_t b);

/* Sparse XOR delta at byte granularity ([XOR] first paragraph): per layer,
 * the ascending int32 positions of the bytes that differ and the new bytes
 * (ref_encode's layout).  Returns the count or -1 (a layer of 2^31 bytes or
 * more). */
int64_t ref_xor_byte_delta(int32_t T, const int64_t *nbytes,
                           const uint8_t *const *old_t, const uint8_t *const *new_t,
                           int64_t *offsets, int32_t *positions, uint8_t *values,
                           int64_t capacity);

/* buf_t[positions[j]] = values[j]; -1 at a position outside its layer. */
int32_t ref_apply_bytes(int32_t T, const int64_t *nbytes, uint8_t *const *buf_t,
                        const int64_t *offsets, const int32_t *positions,
                        const uint8_t *values);

#ifdef __cplusplus
}
#endif

#endif /* DWS_ORACLE_H */
