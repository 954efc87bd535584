/*
 * sconv_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, scalar, double-precision CPU statement of what the fused
 * short-convolution path computes.  It exists only so that the CUDA kernels
 * can be checked against it: only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load it.  It shares no code, header,
 * table or constant with the CUDA library, and the library never calls it.
 *
 * Sources followed (web pages, by title and section):
 *   [P1] "vllm.models.inkling.nvidia.ops.sconv" -- module docstring (paged
 *        sliding-window cache, stream D-sub-range, same-forward vs
 *        pre-forward taps), fused_sconv (argument list and shapes),
 *        sconv_seq_metadata (seq_idx / query_start buffers, padded rows).
 *   [P2] "core.ssm.ops.intermediate_extraction" -- _scatter_intermediate_conv_kernel
 *        and scatter_intermediate_conv (conditional, transposed window gather).
 *   [P4] "Implementation:Sgl project Sglang Mamba Ops" -- causal_conv1d_fwd
 *        and causal_conv1d_update (the same convolution over dense
 *        per-sequence state lines: conv_states, cache_indices,
 *        has_initial_state, bias, pad_slot_id; x and states in place).
 *
 * Readings taken where the pages are silent (each one is a single place in
 * this file):
 *   - tap orientation: weight[c][W-1] multiplies the current position,
 *     weight[c][0] the oldest one (the causal_conv1d convention that [P4]
 *     names); see TAP_POSITION below.
 *   - a tap belongs to this step's forward (and is read from x) when its x
 *     row t + src - pos is at or after query_start[t], the first x row of
 *     the token's request ([P1] fused_sconv argument comments).
 *   - epilogue order: out = act(conv) + x  (activation on the convolution,
 *     residual added after); see EPILOGUE below.
 *   - PAD rows (slot_mapping == -1) produce no output row and no cache write.
 *   - window rows outside [0, seq_len) of an extraction read as zero.
 *   - tokens whose indices fall outside the buffers they address are skipped
 *     whole and counted (the library's documented bounds policy).
 *
 * Everything is computed in double.  Inputs are decoded exactly from their
 * stored type (bf16 by a 16-bit shift into a float, float to double), and
 * cache inserts / window gathers are byte copies.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static size_t elem_bytes(int dtype) { return dtype == ORACLE_F32 ? 4u : 2u; }

/* Exact decode of one stored element to double. */
static double load_value(const void *base, int dtype, int64_t index) {
    if (dtype == ORACLE_F32) {
        float f;
        memcpy(&f, (const char *)base + index * 4, 4);
        return (double)f;
    }
    uint16_t h;
    memcpy(&h, (const char *)base + index * 2, 2);
    uint32_t bits = (uint32_t)h << 16; /* bf16 is the top half of a float */
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

static void copy_element(void *dst, int64_t dst_index, const void *src,
                         int64_t src_index, int dtype) {
    size_t e = elem_bytes(dtype);
    memcpy((char *)dst + dst_index * (int64_t)e,
           (const char *)src + src_index * (int64_t)e, e);
}

/* Reading of the tap orientation: tap k of a W-tap window ending at
 * position pos sits at absolute position pos - (W-1) + k, so tap W-1 is the
 * current token and tap 0 the oldest ([P4] causal_conv1d convention). */
#define TAP_POSITION(pos, W, k) ((pos) - ((W) - 1) + (k))

/* Reading of the epilogue order: activation on the convolution, then the
 * residual input added ([P1] fused_sconv flags activation, use_residual). */
#define EPILOGUE(conv, xv, silu, resid)                                       \
    (((silu) ? (conv) / (1.0 + exp(-(conv))) : (conv)) + ((resid) ? (xv) : 0.0))

enum tap_kind { TAP_X = 0, TAP_ZERO = 1, TAP_CACHE = 2 };

/*
 * oracle_fused -- [P1] fused_sconv: per token, insert x into its cache slot
 * and convolve the W taps ending at its absolute position.
 *
 * Shapes and layouts follow [P1] fused_sconv's argument comments:
 *   x            [T, C]  row stride x_row_stride, element stride 1, C = H*ws
 *   weight       [C, W]  strides (w_stride_c, w_stride_k)
 *   cache        [num_blocks, H, N, D]  strides cache_strides[0..3]
 *   positions    [T] int64   absolute position of each token
 *   seq_idx      [T] int32   request of each token
 *   slot_mapping [T] int64   flat slot block*N + offset; -1 = PAD (skip)
 *   query_start  [T] int32   first x row of the token's request
 *   block_table  [num_reqs, max_blocks] int32, row stride bt_row_stride
 * The stream owns cache lanes [off_s, off_s + ws) of every head; channel
 * c = h*ws + j lives at lane off_s + j of head h.
 *
 * Pre-forward taps are read from cache_in (the cache as it was before the
 * call).  If cache_out is not NULL the inserts of tokens in
 * [t_begin, t_end) are written into it (the caller passes a copy of
 * cache_in).  For every token t in [t_begin, t_end), row t - t_begin of
 * out_ref [t_end - t_begin, C] receives the double-precision result and
 * row_state[t - t_begin] is 1 (computed), 0 (PAD) or 2 (skipped: an index
 * out of range).  If write_index is not NULL, write_index[(t - t_begin)*C + c]
 * receives the flat cache element index that token t's channel c is inserted
 * at, or -1 when the token writes nothing (a sparse record of the inserts
 * for caches too large to copy).  Returns the number of skipped tokens, or
 * -1 if an argument is malformed.
 */
int64_t oracle_fused(int dtype, const void *x, int64_t x_row_stride, int64_t T,
                     int64_t C, const void *weight, int64_t w_stride_c,
                     int64_t w_stride_k, int W, const void *cache_in,
                     void *cache_out, const int64_t *cache_strides,
                     int64_t num_blocks, int64_t H, int64_t N, int64_t D,
                     const int64_t *positions, const int32_t *seq_idx,
                     const int64_t *slot_mapping, const int32_t *query_start,
                     const int32_t *block_table, int64_t bt_row_stride,
                     int64_t num_reqs, int64_t max_blocks, int64_t off_s,
                     int64_t ws, int silu, int residual, int64_t t_begin,
                     int64_t t_end, double *out_ref, uint8_t *row_state,
                     int64_t *write_index) {
    if (W < 1 || C != H * ws || off_s < 0 || off_s + ws > D || N < 1 ||
        t_begin < 0 || t_end > T || t_begin > t_end)
        return -1;
    int64_t skipped = 0;
    enum tap_kind kind[64];
    int64_t tap_block[64];
    if (W > 64) return -1;

    for (int64_t t = t_begin; t < t_end; ++t) {
        int64_t local = t - t_begin;
        row_state[local] = 0;
        if (write_index)
            for (int64_t c = 0; c < C; ++c) write_index[local * C + c] = -1;
        int64_t slot = slot_mapping[t];
        if (slot == -1) continue; /* PAD row: no write, no output ([P1]) */

        int64_t pos = positions[t];
        int64_t req = seq_idx[t];
        int64_t q0 = query_start[t];
        int bad = slot < 0 || slot >= num_blocks * N || req < 0 ||
                  req >= num_reqs || q0 < 0 || q0 > t || pos < 0;

        /* Resolve where each tap comes from ([P1] module docstring). */
        for (int k = 0; k < W && !bad; ++k) {
            int64_t src = TAP_POSITION(pos, W, k);
            int64_t row = t + (src - pos);
            if (row >= q0) {
                kind[k] = TAP_X; /* same-forward tap: x row src - pos + t */
            } else if (src < 0) {
                kind[k] = TAP_ZERO; /* before position 0 */
            } else {
                int64_t logical = src / N;
                if (logical >= max_blocks) { bad = 1; break; }
                int64_t b = block_table[req * bt_row_stride + logical];
                if (b < 0 || b >= num_blocks) { bad = 1; break; }
                kind[k] = TAP_CACHE; /* pre-forward tap via block_table */
                tap_block[k] = b;
            }
        }
        if (bad) {
            row_state[local] = 2;
            ++skipped;
            continue;
        }
        row_state[local] = 1;

        for (int64_t c = 0; c < C; ++c) {
            int64_t h = c / ws, j = c % ws;
            int64_t x_index = t * x_row_stride + c;
            int64_t dst = (slot / N) * cache_strides[0] + h * cache_strides[1] +
                          (slot % N) * cache_strides[2] + (off_s + j) * cache_strides[3];
            if (cache_out) copy_element(cache_out, dst, x, x_index, dtype);
            if (write_index) write_index[local * C + c] = dst;
            double acc = 0.0;
            for (int k = 0; k < W; ++k) {
                int64_t src = TAP_POSITION(pos, W, k);
                double v;
                if (kind[k] == TAP_X) {
                    v = load_value(x, dtype, (t + (src - pos)) * x_row_stride + c);
                } else if (kind[k] == TAP_ZERO) {
                    v = 0.0;
                } else {
                    int64_t idx = tap_block[k] * cache_strides[0] +
                                  h * cache_strides[1] +
                                  (src % N) * cache_strides[2] +
                                  (off_s + j) * cache_strides[3];
                    v = load_value(cache_in, dtype, idx);
                }
                acc += load_value(weight, dtype, c * w_stride_c + k * w_stride_k) * v;
            }
            out_ref[local * C + c] =
                EPILOGUE(acc, load_value(x, dtype, x_index), silu, residual);
        }
    }
    return skipped;
}

/*
 * oracle_seq_metadata -- [P1] sconv_seq_metadata: for every token
 * t < num_actual, seq_idx[t] is the last request r < num_reqs whose start
 * query_start_loc[r] is <= t (so empty requests are never chosen) and
 * query_start[t] = query_start_loc[seq_idx[t]]; rows
 * [num_actual, num_padded) are filled with zero.  A plain linear scan.
 */
void oracle_seq_metadata(const int32_t *query_start_loc, int64_t num_reqs,
                         int64_t num_actual, int64_t num_padded,
                         int32_t *seq_idx_out, int32_t *query_start_out) {
    for (int64_t t = 0; t < num_padded; ++t) {
        if (t >= num_actual) {
            seq_idx_out[t] = 0;
            query_start_out[t] = 0;
            continue;
        }
        int64_t found = 0;
        for (int64_t r = 0; r < num_reqs; ++r)
            if (query_start_loc[r] <= t) found = r;
        seq_idx_out[t] = (int32_t)found;
        query_start_out[t] = query_start_loc[found];
    }
}

/*
 * oracle_resolve_taps -- the tap-source resolution of [P1] (module
 * docstring and fused_sconv argument comments) written out per token, so
 * that it can be done once per step and read by every layer's convolution.
 *
 * The token's request r and first x row q0 come from query_start_loc as in
 * oracle_seq_metadata (last r with query_start_loc[r] <= t), or, when
 * query_start_loc is NULL (the decode form, token t is request t), r = q0 = t.
 * For a non-PAD token t < num_actual at position pos, the entry for lag
 * d = 1..W-1 (the tap at position src = pos - d), taps[t*(W-1) + d-1], is
 *   -2                 the same-forward tap: x row t - d, when t - d >= q0;
 *   -1                 the zero tap: src < 0 (and t - d < q0);
 *   b*N + src % N      otherwise: the flat cache slot of src, with
 *                      b = block_table[r][src / N] (the block/offset split
 *                      of a flat slot that slot_mapping uses);
 *   -(flags * 256)     for every lag, when the token cannot be resolved:
 *                      flags holds the bounds-policy bits of its own
 *                      indices (0x02 request >= num_reqs, 0x10 q0 outside
 *                      [0, t], 0x20 pos < 0) or, when those are clean, the
 *                      union over its cache taps of 0x04 (src / N >=
 *                      max_blocks) and 0x08 (block outside [0, num_blocks)).
 * PAD rows (slot_mapping == -1) and rows [num_actual, num_padded) get -1 at
 * every lag and are never flagged.  seq_idx_out / query_start_out (either
 * may be NULL) receive r and q0, and 0 on rows [num_actual, num_padded).
 */
#define SRC_X (-2)
#define SRC_ZERO (-1)

void oracle_resolve_taps(const int32_t *query_start_loc, int64_t num_reqs,
                         int64_t num_actual, int64_t num_padded,
                         const int64_t *positions, const int64_t *slot_mapping,
                         const int32_t *block_table, int64_t bt_row_stride,
                         int64_t max_blocks, int64_t num_blocks, int64_t N, int W,
                         int32_t *seq_idx_out, int32_t *query_start_out,
                         int64_t *taps) {
    int64_t L = W - 1;
    for (int64_t t = 0; t < num_padded; ++t) {
        int64_t r = 0, q0 = 0;
        for (int64_t d = 1; d <= L; ++d) taps[t * L + d - 1] = SRC_ZERO;
        if (t < num_actual) {
            if (query_start_loc) {
                for (int64_t k = 0; k < num_reqs; ++k)
                    if (query_start_loc[k] <= t) r = k;
                q0 = query_start_loc[r];
            } else {
                r = t;
                q0 = t;
            }
        }
        if (seq_idx_out) seq_idx_out[t] = (int32_t)r;
        if (query_start_out) query_start_out[t] = (int32_t)q0;
        if (t >= num_actual || slot_mapping[t] == -1) continue;

        int64_t pos = positions[t];
        int64_t own = 0;
        if (r >= num_reqs) own |= 0x02;
        if (q0 < 0 || q0 > t) own |= 0x10;
        if (pos < 0) own |= 0x20;
        int64_t flags = own;
        if (!own) {
            for (int64_t d = 1; d <= L; ++d) {
                int64_t src = pos - d;
                int64_t *e = &taps[t * L + d - 1];
                if (t - d >= q0) {
                    *e = SRC_X;            /* same-forward tap ([P1]) */
                } else if (src < 0) {
                    *e = SRC_ZERO;         /* before position 0 */
                } else {
                    int64_t logical = src / N;
                    if (logical >= max_blocks) { flags |= 0x04; continue; }
                    int64_t b = block_table[r * bt_row_stride + logical];
                    if (b < 0 || b >= num_blocks) { flags |= 0x08; continue; }
                    *e = b * N + src % N;  /* pre-forward tap via block_table */
                }
            }
        }
        if (flags)
            for (int64_t d = 1; d <= L; ++d) taps[t * L + d - 1] = -(flags * 256);
    }
}

/*
 * oracle_extract_windows -- [P2] scatter_intermediate_conv: for slot
 * i < real_count, out[i][c][k] = src[abs_positions[i] - d_conv + k][c]
 * (window [pos - d_conv, pos), written transposed), with rows outside
 * [0, seq_len) reading as zero; slots i >= real_count are left untouched.
 * `out` holds the caller's prior bytes on entry.  real_count is clamped to
 * [0, max_count].
 */
void oracle_extract_windows(int dtype, const void *src, int64_t seq_len,
                            int64_t conv_dim, int64_t src_stride_s,
                            int64_t src_stride_c, const int32_t *abs_positions,
                            int64_t real_count, int64_t max_count, void *out,
                            int64_t out_slot_stride, int64_t d_conv) {
    if (real_count > max_count) real_count = max_count;
    size_t e = elem_bytes(dtype);
    for (int64_t i = 0; i < real_count; ++i) {
        for (int64_t c = 0; c < conv_dim; ++c) {
            for (int64_t k = 0; k < d_conv; ++k) {
                int64_t p = (int64_t)abs_positions[i] - d_conv + k;
                int64_t dst = i * out_slot_stride + c * d_conv + k;
                if (p >= 0 && p < seq_len)
                    copy_element(out, dst, src, p * src_stride_s + c * src_stride_c,
                                 dtype);
                else
                    memset((char *)out + dst * (int64_t)e, 0, e);
            }
        }
    }
}

/* ---- precondition checks used by the tests' generator audit ---------- */

static int cmp_i64(const void *a, const void *b) {
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

/*
 * oracle_check_preconditions -- the conditions under which one launch is
 * well defined ([P1] module docstring: the just-written slot is never read
 * back in the same step; a request's rows are contiguous with positions
 * rising by one):
 *   1. within a request, positions[t] - t is constant and seq_idx agrees;
 *   2. non-PAD slots are distinct;
 *   3. no written slot is also read as a pre-forward tap.
 * Returns 0 when all hold, else the number (1..3) of the first one broken.
 */
int oracle_check_preconditions(int64_t T, int W, int64_t N,
                               const int64_t *positions, const int32_t *seq_idx,
                               const int64_t *slot_mapping,
                               const int32_t *query_start,
                               const int32_t *block_table,
                               int64_t bt_row_stride, int64_t max_blocks) {
    for (int64_t t = 0; t < T; ++t) {
        int64_t q0 = query_start[t];
        if (q0 < 0 || q0 > t) return 1;
        if (seq_idx[t] != seq_idx[q0]) return 1;
        if (positions[t] - t != positions[q0] - q0) return 1;
    }
    int64_t *written = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T + 1));
    int64_t *read = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T * W + 1));
    int64_t nw = 0, nr = 0;
    for (int64_t t = 0; t < T; ++t) {
        if (slot_mapping[t] == -1) continue;
        written[nw++] = slot_mapping[t];
        int64_t pos = positions[t];
        for (int k = 0; k < W; ++k) {
            int64_t src = TAP_POSITION(pos, W, k);
            if (t + (src - pos) >= query_start[t] || src < 0) continue;
            int64_t logical = src / N;
            if (logical >= max_blocks) continue;
            int64_t b = block_table[(int64_t)seq_idx[t] * bt_row_stride + logical];
            read[nr++] = b * N + src % N;
        }
    }
    qsort(written, (size_t)nw, sizeof(int64_t), cmp_i64);
    int result = 0;
    for (int64_t i = 1; i < nw && !result; ++i)
        if (written[i] == written[i - 1]) result = 2;
    for (int64_t i = 0; i < nr && !result; ++i)
        if (bsearch(&read[i], written, (size_t)nw, sizeof(int64_t), cmp_i64))
            result = 3;
    free(written);
    free(read);
    return result;
}

/*
 * oracle_scatter_ssm -- [P2] scatter_intermediate_ssm: for slot
 * i < real_count (clamped to [0, max_count]) out row i becomes states row
 * chunk_indices[i] (state_flat elements, a byte copy).  Slots at or beyond
 * real_count, and slots whose index is outside [0, num_chunks), keep their
 * bytes.  Returns the number of slots skipped for a bad index.
 */
int64_t oracle_scatter_ssm(int dtype, const void *states, int64_t num_chunks,
                           int64_t state_flat, int64_t states_row_stride,
                           const int64_t *chunk_indices, int64_t real_count,
                           int64_t max_count, void *out, int64_t out_row_stride) {
    if (real_count > max_count) real_count = max_count;
    int64_t skipped = 0;
    for (int64_t i = 0; i < real_count; ++i) {
        int64_t row = chunk_indices[i];
        if (row < 0 || row >= num_chunks) {
            ++skipped;
            continue;
        }
        for (int64_t e = 0; e < state_flat; ++e)
            copy_element(out, i * out_row_stride + e, states, row * states_row_stride + e,
                         dtype);
    }
    return skipped;
}

/*
 * oracle_extract_windows_paged -- the window gather of
 * oracle_extract_windows with the conv input read from the paged cache of
 * [P1]: for slot i < real_count, request r = request[i] and
 * p = abs_positions[i] - d_conv + k,
 *     out[i][c][k] = cache[block_table[r][p / N], h, p % N, off_s + j]
 * (c = h*ws + j), zero for p < 0.  A slot whose request, logical block or
 * block-table entry is out of range keeps its bytes and is counted.
 */
int64_t oracle_extract_windows_paged(int dtype, const void *cache,
                                     const int64_t *cache_strides, int64_t num_blocks,
                                     int64_t H, int64_t N, int64_t off_s, int64_t ws,
                                     const int32_t *block_table, int64_t bt_row_stride,
                                     int64_t num_reqs, int64_t max_blocks,
                                     const int32_t *request, const int32_t *abs_positions,
                                     int64_t real_count, int64_t max_count, void *out,
                                     int64_t out_slot_stride, int64_t d_conv) {
    if (real_count > max_count) real_count = max_count;
    if (d_conv > 64) return -1;
    size_t e = elem_bytes(dtype);
    int64_t skipped = 0;
    int64_t blk[64];
    for (int64_t i = 0; i < real_count; ++i) {
        int64_t r = request[i];
        int bad = r < 0 || r >= num_reqs;
        for (int64_t k = 0; k < d_conv && !bad; ++k) {
            int64_t p = (int64_t)abs_positions[i] - d_conv + k;
            blk[k] = -1;
            if (p < 0) continue;
            if (p / N >= max_blocks) { bad = 1; break; }
            int64_t b = block_table[r * bt_row_stride + p / N];
            if (b < 0 || b >= num_blocks) { bad = 1; break; }
            blk[k] = b;
        }
        if (bad) {
            ++skipped;
            continue;
        }
        for (int64_t c = 0; c < H * ws; ++c) {
            int64_t h = c / ws, j = c % ws;
            for (int64_t k = 0; k < d_conv; ++k) {
                int64_t p = (int64_t)abs_positions[i] - d_conv + k;
                int64_t dst = i * out_slot_stride + c * d_conv + k;
                if (p < 0) {
                    memset((char *)out + dst * (int64_t)e, 0, e);
                } else {
                    int64_t src = blk[k] * cache_strides[0] + h * cache_strides[1] +
                                  (p % N) * cache_strides[2] + (off_s + j) * cache_strides[3];
                    copy_element(out, dst, cache, src, dtype);
                }
            }
        }
    }
    return skipped;
}

/* ---------------------------------------------------------------------------
 * The dense-state interface of [P4]: causal_conv1d_fwd and
 * causal_conv1d_update, where a sequence's history is a dense state line
 * (conv_states[line]) instead of the paged cache.
 *
 * Reading of the state line: it holds the last L inputs of its sequence,
 * oldest first (entry L-1 is the most recent input), L >= W-1.  A sequence
 * is convolved over its extended input e = (state line, or L zeros) followed
 * by its x rows, so output t uses e entries L + TAP_POSITION(t, W, k), and
 * the line afterwards holds the last L entries of e.
 *
 * Reading of the bias: added to the convolution before the activation.
 */
#define BIASED(conv, b) ((conv) + (b))

/* Element index of entry i of a state line. */
#define STATE_INDEX(line, c, i, s_line, s_c, s_k) \
    ((line) * (s_line) + (c) * (s_c) + (i) * (s_k))

/*
 * oracle_conv1d_fwd -- [P4] causal_conv1d_fwd (varlen prefill).
 *   x        [total_tokens, dim], strides (x_st, x_sc)
 *   weight   [dim, W], strides (w_sc, w_sk);  bias [dim] or NULL
 *   states_in / states_out: [num_lines, dim, L] with strides
 *            (s_line, s_c, s_k); states_out is the caller's copy of
 *            states_in and receives the new lines.  states_in NULL: zero
 *            history, no state write.
 *   qsl      [batch+1] sequence b is x rows qsl[b] .. qsl[b+1]-1
 *   cache_indices [batch] state line of sequence b (NULL: b); a sequence
 *            whose line equals pad_slot_id is skipped
 *   has_init [batch] 1 = start from the state line, 0 = from zeros
 *            (NULL: all 0)
 * out_ref [total_tokens, dim] receives the double results of computed rows;
 * row_state[t] is 1 (computed), 0 (not part of a computed sequence) or 2
 * (skipped: the line is outside [0, num_lines)).  Returns the number of
 * skipped sequences, or -1 if an argument is malformed.
 */
int64_t oracle_conv1d_fwd(int dtype, const void *x, int64_t x_st, int64_t x_sc,
                          int64_t total_tokens, int64_t dim, const void *weight,
                          int64_t w_sc, int64_t w_sk, int W, const void *bias,
                          const void *states_in, void *states_out, int64_t s_line,
                          int64_t s_c, int64_t s_k, int64_t L, int64_t num_lines,
                          const int32_t *qsl, int64_t batch,
                          const int32_t *cache_indices, const uint8_t *has_init,
                          int silu, int64_t pad_slot_id, double *out_ref,
                          uint8_t *row_state) {
    if (W < 1 || batch < 0 || (states_in && (L < W - 1 || !states_out)))
        return -1;
    for (int64_t t = 0; t < total_tokens; ++t) row_state[t] = 0;
    int64_t skipped = 0;
    for (int64_t b = 0; b < batch; ++b) {
        int64_t q0 = qsl[b], q1 = qsl[b + 1];
        if (q0 < 0 || q1 < q0 || q1 > total_tokens) return -1;
        int64_t line = cache_indices ? cache_indices[b] : b;
        if (cache_indices && line == pad_slot_id) continue; /* padded entry */
        if (states_in && (line < 0 || line >= num_lines)) {
            for (int64_t t = q0; t < q1; ++t) row_state[t] = 2;
            ++skipped;
            continue;
        }
        int from_state = states_in && has_init && has_init[b];
        int64_t Lh = states_in ? L : W - 1; /* history entries ahead of x */
        int64_t n = q1 - q0;
        for (int64_t c = 0; c < dim; ++c) {
            for (int64_t t = 0; t < n; ++t) {
                double acc = 0.0;
                for (int k = 0; k < W; ++k) {
                    int64_t i = Lh + TAP_POSITION(t, W, k); /* entry of e */
                    double v;
                    if (i >= Lh)
                        v = load_value(x, dtype, (q0 + i - Lh) * x_st + c * x_sc);
                    else if (from_state)
                        v = load_value(states_in, dtype,
                                       STATE_INDEX(line, c, i, s_line, s_c, s_k));
                    else
                        v = 0.0;
                    acc += load_value(weight, dtype, c * w_sc + k * w_sk) * v;
                }
                double bv = bias ? load_value(bias, dtype, c) : 0.0;
                out_ref[(q0 + t) * dim + c] = EPILOGUE(BIASED(acc, bv), 0.0, silu, 0);
            }
            if (!states_in) continue;
            /* new line = the last L entries of e, i.e. entries n .. n+L-1 */
            for (int64_t i = 0; i < L; ++i) {
                int64_t j = n + i;
                int64_t dst = STATE_INDEX(line, c, i, s_line, s_c, s_k);
                if (j >= Lh)
                    copy_element(states_out, dst, x, (q0 + j - Lh) * x_st + c * x_sc, dtype);
                else if (from_state)
                    copy_element(states_out, dst, states_in,
                                 STATE_INDEX(line, c, j, s_line, s_c, s_k), dtype);
                else
                    memset((char *)states_out + dst * (int64_t)elem_bytes(dtype), 0,
                           elem_bytes(dtype));
            }
        }
        for (int64_t t = q0; t < q1; ++t) row_state[t] = 1;
    }
    return skipped;
}

/*
 * oracle_conv1d_update -- [P4] causal_conv1d_update (one token per
 * sequence).  x [batch, dim] strides (x_sb, x_sc); state lines as in
 * oracle_conv1d_fwd; indices [batch] (NULL: b), pad_slot_id skips.
 *
 * cache_seqlens NULL: the line is shifted -- its entries are the last L
 * inputs, the taps before the token are entries L-(W-1) .. L-1, and the new
 * line is the last L entries of (line, x) -- exactly oracle_conv1d_fwd on a
 * one-row sequence that starts from its state.
 * cache_seqlens given (reading: a circular line): s = cache_seqlens[b] inputs
 * were seen, input at position p is kept at entry p mod L; the taps before
 * the token are positions s-(W-1) .. s-1 and the token is stored at entry
 * s mod L, nothing else moves.
 * out_ref [batch, dim]; row_state[b] 1 computed / 0 padded / 2 bad line.
 */
int64_t oracle_conv1d_update(int dtype, const void *x, int64_t x_sb, int64_t x_sc,
                             int64_t batch, int64_t dim, const void *weight, int64_t w_sc,
                             int64_t w_sk, int W, const void *bias, const void *states_in,
                             void *states_out, int64_t s_line, int64_t s_c, int64_t s_k,
                             int64_t L, int64_t num_lines, const int32_t *cache_seqlens,
                             const int32_t *indices, int silu, int64_t pad_slot_id,
                             double *out_ref, uint8_t *row_state) {
    if (W < 2 || L < W - 1 || !states_in || !states_out) return -1;
    int64_t skipped = 0;
    for (int64_t b = 0; b < batch; ++b) {
        row_state[b] = 0;
        int64_t line = indices ? indices[b] : b;
        if (indices && line == pad_slot_id) continue;
        if (line < 0 || line >= num_lines) {
            row_state[b] = 2;
            ++skipped;
            continue;
        }
        row_state[b] = 1;
        int64_t s = cache_seqlens ? cache_seqlens[b] : 0;
        for (int64_t c = 0; c < dim; ++c) {
            double acc = 0.0;
            for (int k = 0; k < W; ++k) {
                double v;
                if (k == W - 1) {
                    v = load_value(x, dtype, b * x_sb + c * x_sc);
                } else {
                    int64_t i;
                    if (cache_seqlens) {
                        int64_t p = s + TAP_POSITION(0, W, k);
                        i = ((p % L) + L) % L;
                    } else {
                        i = L + TAP_POSITION(0, W, k);
                    }
                    v = load_value(states_in, dtype, STATE_INDEX(line, c, i, s_line, s_c, s_k));
                }
                acc += load_value(weight, dtype, c * w_sc + k * w_sk) * v;
            }
            double bv = bias ? load_value(bias, dtype, c) : 0.0;
            out_ref[b * dim + c] = EPILOGUE(BIASED(acc, bv), 0.0, silu, 0);
            if (cache_seqlens) {
                int64_t i = ((s % L) + L) % L;
                copy_element(states_out, STATE_INDEX(line, c, i, s_line, s_c, s_k), x,
                             b * x_sb + c * x_sc, dtype);
            } else {
                for (int64_t i = 0; i + 1 < L; ++i)
                    copy_element(states_out, STATE_INDEX(line, c, i, s_line, s_c, s_k),
                                 states_in, STATE_INDEX(line, c, i + 1, s_line, s_c, s_k),
                                 dtype);
                copy_element(states_out, STATE_INDEX(line, c, L - 1, s_line, s_c, s_k), x,
                             b * x_sb + c * x_sc, dtype);
            }
        }
    }
    return skipped;
}
