/*
 * sconv.h -- C ABI of the B200 (sm_100a) fused short-convolution library.
 *
 * The operation is the short-convolution step of hybrid attention/SSM
 * inference described on the page "vllm.models.inkling.nvidia.ops.sconv"
 * (module docstring and fused_sconv):
 *
 *   A layer's conv streams share one paged cache [num_blocks, H, N, D]
 *   (head-major).  A stream owns the lanes [off_s, off_s + ws) of every head,
 *   so its per-token channel count is C = H * ws and channel c = h*ws + j
 *   lives at lane off_s + j of head h.  The cache holds the conv input at
 *   every absolute position.  For each token one launch
 *     1. writes the token's input row x[t, :] into its slot
 *        (slot_mapping[t] = block * N + offset; -1 marks a PAD row, skipped);
 *     2. convolves, per channel, the W taps ending at the token's absolute
 *        position: a tap inside the current forward is read from x (row
 *        t + src - pos), an earlier one from the cache through
 *        block_table[request, src / N] at offset src % N, and a tap before
 *        position 0 is zero;
 *     3. applies the optional SiLU to the convolution and then adds the
 *        residual x[t, c];
 *   and is valid for prefill, decode and speculative tokens alike.
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller.  Nothing is
 *     allocated, freed or synchronised: work is enqueued on `stream`, the
 *     grid depends only on the token count and channel count (or on
 *     max_count), so every call can be captured in a CUDA graph.
 *   - Strides are in ELEMENTS.  The innermost stride of x, out, src and the
 *     cache D axis must be 1.
 *   - Floating-point data (x, weight, cache, out, src) all have the one
 *     dtype `dt`.  Accumulation is in fp32 over taps in order k = 0..W-1;
 *     bf16 results are rounded to nearest even once.
 *   - Tap orientation: weight[c][W-1] multiplies the current position and
 *     weight[c][0] the position W-1 steps back (the causal_conv1d convention
 *     of "Implementation:Sgl project Sglang Mamba Ops").
 *   - Arguments are checked on the host before anything is enqueued; a bad
 *     argument returns SCONV_ERR_INVALID or SCONV_ERR_UNSUPPORTED and
 *     enqueues nothing.  The library never aborts the process.
 *   - Indices read on the device (slots, requests, block-table entries,
 *     query starts, positions) are range-checked per token.  A token with an
 *     index out of range is skipped whole (no cache write, no output row)
 *     and, if `err_flag` is not NULL, the matching SCONV_EFLAG_* bits are
 *     OR-ed into *err_flag.  Nothing traps or waits.
 *   - Every kernel is launched with programmatic dependent launch: it may
 *     start while the kernel before it on the stream still runs, and waits
 *     for that kernel to complete before it reads data that kernel may
 *     write.  weight and bias are the exception: they may be read before
 *     that wait, so the kernel that precedes a call on the stream must not
 *     write them.
 *   - Preconditions not checked (behaviour is undefined when broken): the
 *     rows of one request are contiguous in x with positions rising by one;
 *     the non-PAD slots of a call are distinct; no slot written by a call is
 *     also read by it as a pre-forward tap (the module docstring's argument
 *     for why one launch has no write/read hazard).
 */
#ifndef SCONV_H
#define SCONV_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sconv_status {
    SCONV_OK = 0,
    SCONV_ERR_INVALID = 1,     /* malformed argument (size, pointer, stride, overlap) */
    SCONV_ERR_UNSUPPORTED = 2, /* well-formed but outside what is built (dtype, W, d_conv) */
    SCONV_ERR_LAUNCH = 3       /* the CUDA launch itself failed */
} sconv_status;

typedef enum sconv_dtype { SCONV_F32 = 0, SCONV_BF16 = 1 } sconv_dtype;

/* fused_sconv's activation: "silu" and "swish" both select SCONV_ACT_SILU. */
typedef enum sconv_act { SCONV_ACT_NONE = 0, SCONV_ACT_SILU = 1 } sconv_act;

/* Bits OR-ed into *err_flag by a token that is skipped. */
#define SCONV_EFLAG_SLOT        0x01u /* slot_mapping not -1 and outside [0, num_blocks*N) */
#define SCONV_EFLAG_REQUEST     0x02u /* seq_idx outside [0, num_reqs) */
#define SCONV_EFLAG_LOGICAL     0x04u /* src / N >= max_blocks for a pre-forward tap */
#define SCONV_EFLAG_BLOCK       0x08u /* block_table entry outside [0, num_blocks) */
#define SCONV_EFLAG_QUERY_START 0x10u /* query_start[t] outside [0, t] */
#define SCONV_EFLAG_POSITION    0x20u /* positions[t] < 0 */
#define SCONV_EFLAG_TIMEOUT     0x40u /* a block's bulk copies did not arrive within its bounded
                                         wait (1 s of wall time by the GPU's global timer, plus
                                         at most one mbarrier try_wait suspension); that block
                                         wrote nothing further and returned */

/*
 * Entries of the resolved tap table that sconv_seq_metadata_taps writes and
 * sconv_fused_taps reads: one int64 per token and lag d = 1..W-1 (the tap at
 * position pos - d), in row t at column d - 1:
 *   >= 0             the flat cache slot block * N + offset of a pre-forward
 *                    tap (the block/offset split slot_mapping uses);
 *   SCONV_TAP_ZERO   a tap before position 0 (zero);
 *   SCONV_TAP_X      a same-forward tap: x row t - d of the same call;
 *   <= -256          the token cannot be resolved; bits 8.. of the negated
 *                    entry are its SCONV_EFLAG_* bits (the same at every lag).
 */
#define SCONV_TAP_ZERO (-1)
#define SCONV_TAP_X    (-2)

#define SCONV_MAX_W 8      /* taps supported by sconv_fused / sconv_update */
#define SCONV_MAX_STREAMS 4 /* conv streams per sconv_fused_streams call */
#define SCONV_MAX_DCONV 8  /* window length supported by sconv_extract_windows */
#define SCONV_MAX_STATE_LEN 16 /* dense state line of sconv_causal_conv1d_fwd / _update */

/*
 * sconv_fused -- insert + depthwise causal conv1d over the paged cache, one
 * launch ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv).
 *
 *   x              [T, C] input rows, row stride x_row_stride (>= C).  Never
 *                  written.  C must equal H * ws.
 *   weight         [C, W] taps, strides (w_stride_c, w_stride_k).  1 <= W <= 8.
 *   cache          [num_blocks, H, N, D], strides cache_strides[0..3] with
 *                  cache_strides[3] == 1.  Read (pre-forward taps) and
 *                  written (inserts) in place.  N is the block size.
 *   positions      [T] int64 absolute position of each token.
 *   seq_idx        [T] int32 request of each token (a block_table row).
 *   slot_mapping   [T] int64 flat slot block*N + offset; -1 = PAD row (no
 *                  cache write, no output row; its x is still read by the
 *                  later tokens of its request).
 *   query_start    [T] int32 first x row of the token's request.
 *   block_table    [num_reqs, max_blocks] int32, row stride bt_row_stride.
 *   off_s, ws      the stream's lanes [off_s, off_s + ws) within D.
 *   act, use_residual   epilogue: out = act(conv) + (use_residual ? x : 0).
 *   dt             dtype of x, weight, cache and out.
 *   out            [T, C], row stride out_row_stride (>= C).  Must not
 *                  overlap x or the cache.  PAD and skipped rows are left
 *                  untouched.
 *   err_flag       optional device int32; see SCONV_EFLAG_*.
 * T == 0 returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_fused(
    const void *x, int64_t x_row_stride, int T, int C,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W,
    void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    const int64_t *positions, const int32_t *seq_idx, const int64_t *slot_mapping,
    const int32_t *query_start,
    const int32_t *block_table, int64_t bt_row_stride, int num_reqs, int max_blocks,
    int off_s, int ws, sconv_act act, int use_residual, sconv_dtype dt,
    void *out, int64_t out_row_stride, int32_t *err_flag, cudaStream_t stream);

/*
 * One conv stream of a layer for sconv_fused_streams: its input, taps,
 * output, lane range and epilogue, each with the meaning it has in
 * sconv_fused (C = H * ws).
 */
typedef struct sconv_stream_desc {
    const void *x;          /* [T, C], row stride x_row_stride */
    int64_t x_row_stride;
    const void *weight;     /* [C, W], strides (w_stride_c, w_stride_k) */
    int64_t w_stride_c, w_stride_k;
    void *out;              /* [T, C], row stride out_row_stride */
    int64_t out_row_stride;
    int off_s, ws;          /* lanes [off_s, off_s + ws) of every head */
    sconv_act act;
    int use_residual;
} sconv_stream_desc;

/*
 * sconv_fused_streams -- the fused step for several conv streams of one layer
 * that share the paged cache, the tokens and all per-token metadata ("each
 * layer's conv streams share one paged cache", vllm sconv page module
 * docstring), in one call.  The result is exactly that of one sconv_fused per
 * stream: the streams' lane ranges must be pairwise disjoint, so no stream
 * reads or writes another's lanes.  At decode sizes one launch serves all
 * streams (the metadata and block-table reads are shared); at prefill sizes
 * each stream gets its own launch.
 *
 *   streams   HOST array of n_streams (1..SCONV_MAX_STREAMS) descriptors;
 *             read during the call only.  Outputs must not overlap any x,
 *             any other output or the cache.
 *   every other argument as in sconv_fused, shared by all streams.
 * T == 0 returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_fused_streams(
    const sconv_stream_desc *streams, int n_streams, int T, int W,
    void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    const int64_t *positions, const int32_t *seq_idx, const int64_t *slot_mapping,
    const int32_t *query_start,
    const int32_t *block_table, int64_t bt_row_stride, int num_reqs, int max_blocks,
    sconv_dtype dt, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_update -- single-token decode form: token b belongs to request b
 * (seq_idx[b] = query_start[b] = b), so every pre-current tap comes from
 * the cache or is zero.  Same computation as sconv_fused on those metadata
 * (the decode update of causal_conv1d_update, "Implementation:Sgl project
 * Sglang Mamba Ops", over the paged cache of the vllm sconv page).
 *
 *   x [B, C], positions [B], slot_mapping [B] (-1 = PAD), block_table
 *   [B, max_blocks]; every other argument as in sconv_fused.
 * B == 0 returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_update(
    const void *x, int64_t x_row_stride, int B, int C,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W,
    void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    const int64_t *positions, const int64_t *slot_mapping,
    const int32_t *block_table, int64_t bt_row_stride, int max_blocks,
    int off_s, int ws, sconv_act act, int use_residual, sconv_dtype dt,
    void *out, int64_t out_row_stride, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_extract_windows -- conditional, transposed gather of the length-d_conv
 * conv windows that prefix caching snapshots ("core.ssm.ops.intermediate_extraction",
 * scatter_intermediate_conv and _scatter_intermediate_conv_kernel).
 *
 *   src            [seq_len, conv_dim], strides (src_stride_s, src_stride_c),
 *                  src_stride_c == 1 (the pre-conv input of one sequence).
 *   abs_positions  [max_count] int32 end position of each slot's window; the
 *                  window is rows [pos - d_conv, pos).  Rows outside
 *                  [0, seq_len) read as zero.
 *   real_count     DEVICE int32[1]: slots i < *real_count are written, slots
 *                  i >= *real_count return at once without touching out.
 *                  The value is clamped to [0, max_count].  Read on the
 *                  device, so the count may change between graph replays.
 *   out            [max_count, conv_dim, d_conv]: out[i][c][k] at
 *                  i*out_slot_stride + c*d_conv + k.  Must not overlap src.
 *   d_conv         1..SCONV_MAX_DCONV.
 * max_count == 0 returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_extract_windows(
    const void *src, int64_t seq_len, int conv_dim, int64_t src_stride_s,
    int64_t src_stride_c, const int32_t *abs_positions, const int32_t *real_count,
    int max_count, void *out, int64_t out_slot_stride, int d_conv, sconv_dtype dt,
    cudaStream_t stream);

/*
 * sconv_scatter_intermediate_ssm -- conditional row gather of SSM chunk-scan
 * states for prefix caching ("core.ssm.ops.intermediate_extraction",
 * _scatter_intermediate_ssm_kernel / scatter_intermediate_ssm): for slot
 * i < *real_count, out row i = states row chunk_indices[i] (state_flat
 * elements); slots i >= *real_count are left untouched and move no data.
 *
 *   states         [num_chunks, state_flat], row stride states_row_stride
 *                  (elements), rows contiguous.
 *   chunk_indices  [max_count] int64 per-slot row index.
 *   real_count     DEVICE int32[1], clamped to [0, max_count], read on the
 *                  device (may change between graph replays).
 *   out            [max_count, state_flat], row stride out_row_stride; must
 *                  not overlap states.
 *   err_flag       optional device int32: a slot whose index is outside
 *                  [0, num_chunks) is left untouched and sets
 *                  SCONV_EFLAG_REQUEST.
 * The copy is bit-exact (dt only fixes the element size).  max_count == 0
 * returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_scatter_intermediate_ssm(
    const void *states, int64_t num_chunks, int64_t state_flat, int64_t states_row_stride,
    const int64_t *chunk_indices, const int32_t *real_count, int max_count, void *out,
    int64_t out_row_stride, sconv_dtype dt, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_extract_windows_paged -- the window extraction of
 * sconv_extract_windows with the conv input read from the paged cache of
 * the vllm sconv page instead of a dense source: for slot i < *real_count,
 * out[i][c][k] = cache[block_table[req, p / N], h, p % N, off_s + j] with
 * req = request[i], p = abs_positions[i] - d_conv + k, c = h*ws + j, and
 * zero for p < 0.  Slots i >= *real_count are untouched.
 *
 *   cache, cache_strides, num_blocks, H, N, D, off_s, ws: as in sconv_fused.
 *   block_table    [num_reqs, max_blocks] int32, row stride bt_row_stride.
 *   request        [max_count] int32 block-table row of each slot.
 *   abs_positions  [max_count] int32 window end (exclusive) of each slot.
 *   real_count     DEVICE int32[1], clamped to [0, max_count].
 *   out            [max_count, C, d_conv] (C = H * ws), out[i][c][k] at
 *                  i*out_slot_stride + c*d_conv + k; must not overlap the cache.
 *   err_flag       optional: a slot whose request or block-table entry is
 *                  out of range is left untouched and sets SCONV_EFLAG_REQUEST,
 *                  SCONV_EFLAG_LOGICAL or SCONV_EFLAG_BLOCK.
 * d_conv in 1..SCONV_MAX_DCONV.  max_count == 0 returns SCONV_OK.
 */
sconv_status sconv_extract_windows_paged(
    const void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    int off_s, int ws, const int32_t *block_table, int64_t bt_row_stride, int num_reqs,
    int max_blocks, const int32_t *request, const int32_t *abs_positions,
    const int32_t *real_count, int max_count, void *out, int64_t out_slot_stride, int d_conv,
    sconv_dtype dt, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_causal_conv1d_fwd -- varlen prefill over dense per-sequence state
 * lines: the interface of causal_conv1d_fwd ("Implementation:Sgl project
 * Sglang Mamba Ops", Signature and I/O Contract).  The same depthwise causal
 * convolution as sconv_fused, with a sequence's history kept as a dense
 * line of its last state_len inputs instead of a paged cache.
 *
 * For sequence b (x rows query_start_loc[b] .. query_start_loc[b+1]-1, n of
 * them) with line = cache_indices[b] (b when cache_indices is NULL):
 *   - line == pad_slot_id (only when cache_indices is given): the sequence is
 *     skipped; its out rows and its line are untouched;
 *   - e = conv_states[line] (state_len entries, oldest first) when
 *     has_initial_state[b] is 1, else state_len zeros, followed by the n x
 *     rows (with conv_states NULL: W-1 zeros followed by the x rows);
 *   - out row t = act(sum_k weight[c][k] * e[t + k + state_len - (W-1)] +
 *     bias[c]): weight[c][W-1] multiplies the current row;
 *   - conv_states[line] = the last state_len entries of e (with n == 0 and
 *     has_initial_state 0 that is a line of zeros).
 *
 *   x                [total_tokens, dim], element strides (x_stride_t,
 *                    x_stride_c): token-major (x_stride_c == 1) or
 *                    channel-major (x_stride_t == 1) storage, or any other
 *                    layout whose elements do not overlap.
 *   weight           [dim, W], strides (w_stride_c, w_stride_k); 2 <= W <= 8.
 *   bias             [dim] contiguous, or NULL.
 *   conv_states      [num_lines, dim, state_len], strides (s_stride_line,
 *                    s_stride_c, s_stride_k), read and written in place; or
 *                    NULL (no history, nothing written).
 *                    W-1 <= state_len <= SCONV_MAX_STATE_LEN.
 *   query_start_loc  [batch+1] int32, 0 <= q[b] <= q[b+1] <= total_tokens.
 *   cache_indices    [batch] int32, or NULL.  Lines of different sequences
 *                    must differ.
 *   has_initial_state [batch] uint8 0/1 (a torch bool tensor), or NULL (0).
 *   out              [total_tokens, dim] with x's strides: either x itself
 *                    (the page's in-place form) or a buffer that does not
 *                    overlap x.  Rows of no computed sequence are untouched.
 *   All floating data (x, weight, bias, conv_states, out) has type dt.
 *   err_flag         optional device int32: a sequence whose line is outside
 *                    [0, num_lines) sets SCONV_EFLAG_SLOT, one whose
 *                    query_start_loc entries are out of order or range sets
 *                    SCONV_EFLAG_QUERY_START; such a sequence is skipped.
 *                    The token-major tiled form (x_stride_c == 1, 16-byte
 *                    aligned rows) sets SCONV_EFLAG_TIMEOUT when a tile's
 *                    copy does not arrive within its bounded wait.
 * One thread block (or warp) owns a (sequence, channel) column and walks it
 * in row order, so the in-place form needs no scratch memory and no ordering
 * between blocks.  weight and bias are read before the wait for the kernel
 * that precedes the call on the stream (programmatic dependent launch), so
 * that kernel must not write them.  Asynchronous; no allocation; CUDA-graph
 * capturable.
 */
sconv_status sconv_causal_conv1d_fwd(
    void *x, int64_t x_stride_t, int64_t x_stride_c, int total_tokens, int dim,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W, const void *bias,
    void *conv_states, int64_t s_stride_line, int64_t s_stride_c, int64_t s_stride_k,
    int state_len, int num_lines, const int32_t *query_start_loc, int batch,
    const int32_t *cache_indices, const uint8_t *has_initial_state, sconv_act act,
    int pad_slot_id, void *out, sconv_dtype dt, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_causal_conv1d_update -- one decode token per sequence over dense
 * state lines: the interface of causal_conv1d_update ("Implementation:Sgl
 * project Sglang Mamba Ops").  For sequence b with line =
 * conv_state_indices[b] (b when NULL; skipped when it equals pad_slot_id):
 *   - cache_seqlens NULL (shifted line): the taps before the token are line
 *     entries state_len-(W-1) .. state_len-1; afterwards the line holds its
 *     last state_len-1 entries followed by x[b] -- exactly
 *     sconv_causal_conv1d_fwd on a one-row sequence with has_initial_state 1;
 *   - cache_seqlens given (circular line): s = cache_seqlens[b] inputs were
 *     seen, the input at position p sits at entry p mod state_len, the taps
 *     before the token are positions s-(W-1) .. s-1, and x[b] is stored at
 *     entry s mod state_len, nothing else moving;
 *   out[b, c] = act(sum_k weight[c][k] * tap_k + bias[c]), tap_{W-1} = x[b, c].
 *
 *   x [batch, dim] (strides x_stride_b, x_stride_c); out has x's strides and
 *   is x itself or does not overlap it.  conv_state is required.  Other
 *   arguments, errors and the rule on weight and bias as in
 *   sconv_causal_conv1d_fwd.
 */
sconv_status sconv_causal_conv1d_update(
    void *x, int64_t x_stride_b, int64_t x_stride_c, int batch, int dim,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W, const void *bias,
    void *conv_state, int64_t s_stride_line, int64_t s_stride_c, int64_t s_stride_k,
    int state_len, int num_lines, const int32_t *cache_seqlens,
    const int32_t *conv_state_indices, sconv_act act, int pad_slot_id, void *out,
    sconv_dtype dt, int32_t *err_flag, cudaStream_t stream);

/*
 * sconv_seq_metadata -- fill the per-token request index and request start
 * in one launch ("vllm.models.inkling.nvidia.ops.sconv", sconv_seq_metadata).
 *
 *   query_start_loc  [num_reqs + 1] int32, non-decreasing, query_start_loc[0] == 0.
 *   For t < num_actual_tokens:
 *       seq_idx_out[t]     = the last r < num_reqs with query_start_loc[r] <= t
 *                            (so an empty request is never chosen);
 *       query_start_out[t] = query_start_loc[seq_idx_out[t]].
 *   Rows [num_actual_tokens, num_padded_tokens) are set to 0 (such rows must
 *   carry slot_mapping == -1 in the sconv_fused call that follows).
 *   num_padded_tokens < 0 means num_padded_tokens = num_actual_tokens.
 *   Returns SCONV_ERR_INVALID (and enqueues nothing) if num_padded_tokens <
 *   num_actual_tokens, or if it exceeds seq_idx_cap or query_start_cap (the
 *   element capacities of the two output buffers), or if num_reqs < 1 while
 *   num_actual_tokens > 0.
 */
sconv_status sconv_seq_metadata(
    const int32_t *query_start_loc, int num_reqs, int num_actual_tokens,
    int num_padded_tokens, int32_t *seq_idx_out, int64_t seq_idx_cap,
    int32_t *query_start_out, int64_t query_start_cap, cudaStream_t stream);

/*
 * sconv_seq_metadata_ahead -- sconv_seq_metadata (same arguments, results
 * and errors) with its work moved ahead of its wait on the stream.
 *
 *   Every launch of this library may start while the kernel before it on
 *   the stream still runs (programmatic dependent launch) and waits for
 *   that kernel's completion before it touches data.  This one reads
 *   query_start_loc and writes both outputs BEFORE that wait and waits
 *   only at its end: it still completes after everything before it on the
 *   stream, so the kernels after it see the usual order, and the lookup
 *   leaves the critical path of back-to-back decode steps.
 *
 *   Precondition (the caller's; nothing checks it): no kernel enqueued
 *   before this call since the stream was last fully ordered (a host
 *   synchronisation, the start of a graph replay) writes query_start_loc or
 *   reads or writes seq_idx_out or query_start_out.  A serving loop meets it
 *   with one metadata buffer set per step in flight, written only by that
 *   step's own call.  Otherwise use sconv_seq_metadata.
 */
sconv_status sconv_seq_metadata_ahead(
    const int32_t *query_start_loc, int num_reqs, int num_actual_tokens,
    int num_padded_tokens, int32_t *seq_idx_out, int64_t seq_idx_cap,
    int32_t *query_start_out, int64_t query_start_cap, cudaStream_t stream);

/*
 * sconv_seq_metadata_taps -- sconv_seq_metadata together with the resolution
 * of every token's pre-forward taps into a table, in one launch.  The
 * resolution is the tap rule of the vllm sconv page (module docstring and
 * fused_sconv): a tap inside the current forward is read from x, an earlier
 * one from the cache through block_table[req, src / N] at offset src % N, a
 * tap before position 0 is zero.  Done once per step, the table serves every
 * layer whose cache shares the block table and block size, and lets
 * sconv_fused_taps reach a token's taps in one dependent memory access
 * instead of three (metadata, block table, cache).
 *
 *   query_start_loc  [num_reqs + 1] int32 as in sconv_seq_metadata, or NULL
 *                    for the decode form: token t is request t.
 *   num_reqs         the requests (query_start_loc given) or the rows of
 *                    block_table (decode form; a token t >= num_reqs is
 *                    flagged SCONV_EFLAG_REQUEST).
 *   positions        [num_actual_tokens] int64 absolute positions.
 *   slot_mapping     [num_actual_tokens] int64; a PAD row (-1) is resolved
 *                    to SCONV_TAP_ZERO at every lag and never flagged.
 *   block_table      [num_reqs, max_blocks] int32, row stride bt_row_stride.
 *   num_blocks, N    the cache's block count and block size.
 *   W                taps, 1..SCONV_MAX_W (W == 1: no table, taps_out may be NULL).
 *   seq_idx_out, query_start_out   as in sconv_seq_metadata (request index
 *                    and its first row; t for both in the decode form);
 *                    either may be NULL and is then not written.
 *   taps_out         [num_padded_tokens, W - 1] int64, row-major, entries as
 *                    SCONV_TAP_* describes; taps_cap is its element capacity.
 *                    Rows [num_actual, num_padded) get SCONV_TAP_ZERO.
 * A token whose own indices are out of range (request, query start,
 * position < 0) gets those bits at every lag; otherwise, if a pre-forward
 * tap lies past the table (src / N >= max_blocks) or on a block outside
 * [0, num_blocks), it gets the union of those bits.
 * Returns SCONV_ERR_INVALID (enqueuing nothing) for negative counts,
 * num_padded_tokens < num_actual_tokens, capacities too small, a missing
 * pointer that is needed, bt_row_stride < max_blocks, or num_reqs < 1 while
 * num_actual_tokens > 0; SCONV_ERR_UNSUPPORTED for W outside 1..8.
 * num_padded_tokens < 0 means num_actual_tokens; 0 rows enqueue nothing.
 */
sconv_status sconv_seq_metadata_taps(
    const int32_t *query_start_loc, int num_reqs, int num_actual_tokens,
    int num_padded_tokens, const int64_t *positions, const int64_t *slot_mapping,
    const int32_t *block_table, int64_t bt_row_stride, int max_blocks, int64_t num_blocks,
    int N, int W, int32_t *seq_idx_out, int64_t seq_idx_cap, int32_t *query_start_out,
    int64_t query_start_cap, int64_t *taps_out, int64_t taps_cap, cudaStream_t stream);

/*
 * sconv_seq_metadata_taps_ahead -- sconv_seq_metadata_taps (same arguments,
 * results and errors) with its work moved ahead of its wait on the stream,
 * as sconv_seq_metadata_ahead does for sconv_seq_metadata, and under the
 * same precondition, extended to every buffer it reads and writes: no
 * kernel enqueued before this call since the stream was last fully ordered
 * writes query_start_loc, positions, slot_mapping or block_table, or reads
 * or writes the three outputs.
 */
sconv_status sconv_seq_metadata_taps_ahead(
    const int32_t *query_start_loc, int num_reqs, int num_actual_tokens,
    int num_padded_tokens, const int64_t *positions, const int64_t *slot_mapping,
    const int32_t *block_table, int64_t bt_row_stride, int max_blocks, int64_t num_blocks,
    int N, int W, int32_t *seq_idx_out, int64_t seq_idx_cap, int32_t *query_start_out,
    int64_t query_start_cap, int64_t *taps_out, int64_t taps_cap, cudaStream_t stream);

/*
 * sconv_fused_taps -- the fused step of sconv_fused_streams (one or more
 * conv streams of a layer; n_streams == 1 is plain sconv_fused) with every
 * token's tap sources read from the table sconv_seq_metadata_taps built for
 * the same step, instead of from positions, seq_idx, query_start and the
 * block table ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv).  The
 * outputs, cache inserts and err_flag bits are bit for bit those of
 * sconv_fused_streams on the metadata the table was built from.
 *
 *   streams, n_streams, T, W, cache, cache_strides, num_blocks, H, N, D, dt:
 *                    as in sconv_fused_streams.
 *   slot_mapping     [T] int64 as in sconv_fused.
 *   taps             [T, W - 1] int64 table built with the same W and N;
 *                    may be NULL when W == 1.  Must not overlap any out.
 *   metadata_ready   0: slot_mapping and taps are read after the wait for
 *                    the kernels this launch depends on (always valid;
 *                    before the wait the table may be read speculatively,
 *                    only to prefetch cache taps into L2).
 *                    1: they are read BEFORE that wait, and each token's x
 *                    rows and cache taps are prefetched into L2 there, so
 *                    that after the wait a token's loads are one dependent
 *                    access.  A launch of this library may begin as soon as
 *                    every kernel it depends on has signalled its
 *                    dependents, which every kernel here except the *_ahead
 *                    builders does after its own wait.  Precondition of 1
 *                    (the caller's; nothing checks it): every kernel that
 *                    writes slot_mapping or taps has completed before any
 *                    kernel this launch depends on could signal it.  Valid
 *                    patterns: the tables were complete before the stream
 *                    (or the graph replay) last started from a fully
 *                    ordered state; or at least one call of this library
 *                    other than the *_ahead builders runs on this stream
 *                    between the builder and this call, and this call
 *                    depends on nothing else.  NOT sufficient: a builder on
 *                    another stream joined by an event -- under stream
 *                    capture that edge becomes programmatic like the
 *                    stream's own, and orders this launch only after the
 *                    builder signals, which is at its start.
 *   err_flag         optional: a skipped token sets the bits its table row
 *                    carries, or SCONV_EFLAG_SLOT (with the row's request,
 *                    query-start and position bits) for a slot out of range;
 *                    an entry that is neither a slot below num_blocks * N,
 *                    SCONV_TAP_X on a row of this call, SCONV_TAP_ZERO nor a
 *                    failure code sets SCONV_EFLAG_BLOCK.
 * Decode-size steps run one thread per 16-byte channel pack of a token.
 * Prefill-size steps of one stream (16-byte aligned x and slot_mapping
 * and taps rows, T >= 64 and T * C / (16 / element size) >= 2^19) run the
 * TMA-pipelined kernel of sconv_fused, whose tiles carry the tokens' table
 * rows instead of their paged metadata; every read then follows the wait
 * (metadata_ready changes nothing there), the outputs, inserts and index
 * bits are the same, and err_flag may also get SCONV_EFLAG_TIMEOUT (a
 * tile's copies did not arrive within the bounded wait).
 * T == 0 returns SCONV_OK and enqueues nothing.
 */
sconv_status sconv_fused_taps(
    const sconv_stream_desc *streams, int n_streams, int T, int W,
    void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    const int64_t *slot_mapping, const int64_t *taps, int metadata_ready, sconv_dtype dt,
    int32_t *err_flag, cudaStream_t stream);

/*
 * One step's tap resolution for sconv_fused_taps_next: the arguments of
 * sconv_seq_metadata_taps for that step, with num_blocks, N and W taken from
 * the sconv_fused_taps_next call.
 */
typedef struct sconv_taps_build {
    const int32_t *query_start_loc;   /* [num_reqs + 1], or NULL (decode form) */
    int num_reqs, num_actual_tokens, num_padded_tokens; /* num_padded < 0: num_actual */
    const int64_t *positions;         /* [num_actual_tokens] */
    const int64_t *slot_mapping;      /* [num_actual_tokens] */
    const int32_t *block_table;       /* [num_reqs, max_blocks] */
    int64_t bt_row_stride;
    int max_blocks;
    int32_t *seq_idx_out;             /* may be NULL */
    int64_t seq_idx_cap;
    int32_t *query_start_out;         /* may be NULL */
    int64_t query_start_cap;
    int64_t *taps_out;                /* [num_padded_tokens, W - 1] */
    int64_t taps_cap;
} sconv_taps_build;

/*
 * sconv_fused_taps_next -- one decode-loop step in one launch: the fused
 * step of sconv_fused_taps for this step (metadata_ready 0: its table is read
 * after the wait for the kernels this launch depends on) and, by extra
 * blocks of the same launch, the tap resolution of sconv_seq_metadata_taps
 * for the NEXT step (`next`).  Those blocks read only the next step's inputs
 * and write only its outputs, so they start at once, never wait and do not
 * hold back the launch of the calls that follow; a following call still
 * waits for this whole launch before it reads the table built here.  So a
 * loop of calls, each building the table the next one reads, keeps the
 * tap resolution off the dependent path of its convolutions, with one launch
 * per step (the first step's table comes from sconv_seq_metadata_taps).
 *
 *   every argument up to err_flag: as in sconv_fused_taps.
 *   next     the next step's resolution; must not be NULL.  Its taps_out
 *            must not overlap `taps` or any out; the same preconditions as
 *            sconv_seq_metadata_taps_ahead apply to its buffers (no kernel
 *            that may still be running writes its inputs or touches its
 *            outputs).
 * Errors: those of sconv_fused_taps and of sconv_seq_metadata_taps for
 * `next`.  T == 0 is allowed (the launch then only builds the next table);
 * T == 0 with next->num_padded_tokens == 0 returns SCONV_OK and enqueues
 * nothing.
 */
sconv_status sconv_fused_taps_next(
    const sconv_stream_desc *streams, int n_streams, int T, int W,
    void *cache, const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
    const int64_t *slot_mapping, const int64_t *taps, sconv_dtype dt, int32_t *err_flag,
    const sconv_taps_build *next, cudaStream_t stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *sconv_status_string(sconv_status status);

/* ABI version of this header; bumped on any incompatible change. */
#define SCONV_ABI_VERSION 1
int sconv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SCONV_H */
