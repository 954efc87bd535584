// api.cu -- the extern "C" entry points declared in include/sconv.h.
//
// Every entry point validates its arguments on the host before it touches
// the CUDA runtime, so a malformed call returns a status and enqueues
// nothing.  Then it picks the 16-byte pack path when every pointer, stride
// and lane offset allows it (else the one-element path) and launches.
#include <limits.h>
#include <stdint.h>

#include "common.cuh"
#include "sconv.h"

namespace {

using sconv::FusedArgs;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t elem_size(sconv_dtype dt) { return dt == SCONV_F32 ? 4 : 2; }

// Half-open byte ranges [lo, hi) overlap?
inline bool overlaps(const void *a, int64_t a_bytes, const void *b, int64_t b_bytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(b_bytes) && b0 < a0 + static_cast<uintptr_t>(a_bytes);
}

// Shared checks of sconv_fused and sconv_update.  Returns SCONV_OK or the
// status to report; on success fills `a` (except the metadata pointers
// specific to one entry point) and `vec`.
sconv_status check_fused(const void *x, int64_t x_rs, int T, int C, const void *weight,
                         int64_t w_sc, int64_t w_sk, int W, void *cache, const int64_t *cs,
                         int64_t num_blocks, int H, int N, int D, const int64_t *positions,
                         const int64_t *slot_mapping, const int32_t *block_table, int64_t bt_rs,
                         int num_reqs, int max_blocks, int off_s, int ws, sconv_act act,
                         int use_residual, sconv_dtype dt, void *out, int64_t out_rs,
                         int32_t *err_flag, FusedArgs &a, bool &vec, bool paged = true) {
    if (dt != SCONV_F32 && dt != SCONV_BF16) return SCONV_ERR_UNSUPPORTED;
    if (W < 1) return SCONV_ERR_INVALID;
    if (W > SCONV_MAX_W) return SCONV_ERR_UNSUPPORTED;
    if (act != SCONV_ACT_NONE && act != SCONV_ACT_SILU) return SCONV_ERR_INVALID;
    if (C < 1 || H < 1 || N < 1 || D < 1 || ws < 1 || off_s < 0) return SCONV_ERR_INVALID;
    if (static_cast<int64_t>(off_s) + ws > D) return SCONV_ERR_INVALID;
    if (static_cast<int64_t>(H) * ws != C) return SCONV_ERR_INVALID;
    if (num_blocks < 1) return SCONV_ERR_INVALID;
    if (!x || !weight || !cache || !cs || !slot_mapping || !out) return SCONV_ERR_INVALID;
    // paged: the call reads positions and the block table itself (every
    // form but sconv_fused_taps, whose taps come resolved)
    if (paged && (num_reqs < 1 || max_blocks < 1 || !positions || !block_table ||
                  bt_rs < max_blocks))
        return SCONV_ERR_INVALID;
    if (cs[3] != 1 || cs[0] < 1 || cs[1] < 1 || cs[2] < 1) return SCONV_ERR_INVALID;
    if (x_rs < C || out_rs < C) return SCONV_ERR_INVALID;
    if (w_sc < 0 || w_sk < 0) return SCONV_ERR_INVALID;

    const int64_t e = elem_size(dt);
    const int64_t x_bytes = ((static_cast<int64_t>(T) - 1) * x_rs + C) * e;
    const int64_t out_bytes = ((static_cast<int64_t>(T) - 1) * out_rs + C) * e;
    const int64_t cache_bytes =
        ((num_blocks - 1) * cs[0] + static_cast<int64_t>(H - 1) * cs[1] +
         static_cast<int64_t>(N - 1) * cs[2] + D) * e;
    if (overlaps(out, out_bytes, x, x_bytes) || overlaps(out, out_bytes, cache, cache_bytes))
        return SCONV_ERR_INVALID;

    const int64_t V = 16 / e;
    vec = aligned16(x) && aligned16(out) && aligned16(cache) && x_rs % V == 0 &&
          out_rs % V == 0 && cs[0] % V == 0 && cs[1] % V == 0 && cs[2] % V == 0 &&
          off_s % V == 0 && ws % V == 0;

    a.x = x;
    a.x_rs = x_rs;
    a.T = T;
    a.C = C;
    a.w = weight;
    a.w_sc = w_sc;
    a.w_sk = w_sk;
    a.W = W;
    a.w_vec = (w_sc == W && w_sk == 1 && aligned16(weight)) ? 1 : 0;
    a.cache = cache;
    a.cs0 = cs[0];
    a.cs1 = cs[1];
    a.cs2 = cs[2];
    a.num_blocks = num_blocks;
    a.H = H;
    a.N = N;
    a.D = D;
    a.positions = positions;
    a.seq_idx = nullptr;
    a.slot = slot_mapping;
    a.qstart = nullptr;
    a.bt = block_table;
    a.bt_rs = bt_rs;
    a.num_reqs = num_reqs;
    a.max_blocks = max_blocks;
    a.off_s = off_s;
    a.ws = ws;
    a.silu = act == SCONV_ACT_SILU;
    a.resid = use_residual != 0;
    a.out = out;
    a.out_rs = out_rs;
    a.err = err_flag;
    a.taps = nullptr;
    return SCONV_OK;
}

// Elements spanned by a strided tensor: the largest offset + 1 (0 if empty).
int64_t span(const int64_t *ext, const int64_t *str, int nd) {
    int64_t last = 0;
    for (int i = 0; i < nd; ++i) {
        if (ext[i] == 0) return 0;
        last += (ext[i] - 1) * str[i];
    }
    return last + 1;
}

// True when no two index tuples of the strided tensor address the same
// element: taken by increasing stride, every dimension of extent > 1 steps
// past everything the smaller dimensions span.
bool non_overlapping(const int64_t *ext, const int64_t *str, int nd) {
    int order[4] = {0, 1, 2, 3};
    for (int i = 0; i < nd; ++i) {
        if (str[i] < 0) return false;
        for (int j = i; j > 0 && str[order[j]] < str[order[j - 1]]; --j) {
            const int t = order[j];
            order[j] = order[j - 1];
            order[j - 1] = t;
        }
    }
    int64_t covered = 1;  // elements spanned by the dimensions taken so far
    for (int i = 0; i < nd; ++i) {
        const int d = order[i];
        if (ext[d] <= 1) continue;
        if (str[d] < covered) return false;
        covered = str[d] * (ext[d] - 1) + covered;
    }
    return true;
}

// Shared checks of the dense-state entry points (T rows of x: the tokens of
// the prefill, the sequences of the update).  Fills `a` and `vec`.
sconv_status check_dense(const void *x, int64_t x_st, int64_t x_sc, int T, int dim,
                         const void *weight, int64_t w_sc, int64_t w_sk, int W, const void *bias,
                         void *states, int64_t s_line, int64_t s_c, int64_t s_k, int L,
                         int num_lines, sconv_act act, void *out, sconv_dtype dt,
                         sconv::DenseArgs &a, bool &vec) {
    if (dt != SCONV_F32 && dt != SCONV_BF16) return SCONV_ERR_UNSUPPORTED;
    if (act != SCONV_ACT_NONE && act != SCONV_ACT_SILU) return SCONV_ERR_INVALID;
    if (W < 2) return SCONV_ERR_INVALID;
    if (W > SCONV_MAX_W) return SCONV_ERR_UNSUPPORTED;
    if (T < 0 || dim < 1 || !x || !weight || !out) return SCONV_ERR_INVALID;
    if (w_sc < 0 || w_sk < 0) return SCONV_ERR_INVALID;
    if (static_cast<int64_t>(dim) > 65535LL * 128) return SCONV_ERR_UNSUPPORTED;
    const int64_t e = elem_size(dt);
    const int64_t xe[2] = {T, dim}, xs[2] = {x_st, x_sc};
    if (!non_overlapping(xe, xs, 2)) return SCONV_ERR_INVALID;
    const int64_t x_bytes = span(xe, xs, 2) * e;
    if (out != x && overlaps(out, x_bytes, x, x_bytes)) return SCONV_ERR_INVALID;
    const int64_t we[2] = {dim, W}, wst[2] = {w_sc, w_sk};
    const int64_t w_bytes = span(we, wst, 2) * e;
    if (overlaps(weight, w_bytes, out, x_bytes)) return SCONV_ERR_INVALID;
    if (bias && overlaps(bias, dim * e, out, x_bytes)) return SCONV_ERR_INVALID;
    if (states) {
        if (L < W - 1) return SCONV_ERR_INVALID;
        if (L > SCONV_MAX_STATE_LEN) return SCONV_ERR_UNSUPPORTED;
        if (num_lines < 1) return SCONV_ERR_INVALID;
        const int64_t se[3] = {num_lines, dim, L}, ss[3] = {s_line, s_c, s_k};
        if (!non_overlapping(se, ss, 3)) return SCONV_ERR_INVALID;
        const int64_t s_bytes = span(se, ss, 3) * e;
        if (overlaps(states, s_bytes, x, x_bytes) || overlaps(states, s_bytes, out, x_bytes) ||
            overlaps(states, s_bytes, weight, w_bytes) ||
            (bias && overlaps(states, s_bytes, bias, dim * e)))
            return SCONV_ERR_INVALID;
    }
    const int64_t V = 16 / e;
    vec = x_sc == 1 && aligned16(x) && aligned16(out) && (x_st * e) % 16 == 0 && dim % V == 0 &&
          dim / V <= 65535;
    a = sconv::DenseArgs{};
    a.x = x;
    a.out = out;
    a.x_st = x_st;
    a.x_sc = x_sc;
    a.T = T;
    a.dim = dim;
    a.w = weight;
    a.w_sc = w_sc;
    a.w_sk = w_sk;
    a.W = W;
    a.bias = bias;
    a.st = states;
    a.s_line = s_line;
    a.s_c = s_c;
    a.s_k = s_k;
    a.L = states ? L : 0;
    a.num_lines = states ? num_lines : 0;
    a.silu = act == SCONV_ACT_SILU;
    a.st_mode = 0;
    if (states && vec && aligned16(states) && (s_line * e) % 16 == 0) {
        if (s_c == 1 && (s_k * e) % 16 == 0)
            a.st_mode = 1;
        else if (s_k == 1 && s_c == L)
            a.st_mode = 2;
    }
    return SCONV_OK;
}

}  // namespace

extern "C" {

int sconv_abi_version(void) { return SCONV_ABI_VERSION; }

const char *sconv_status_string(sconv_status s) {
    switch (s) {
        case SCONV_OK: return "ok";
        case SCONV_ERR_INVALID: return "invalid argument";
        case SCONV_ERR_UNSUPPORTED: return "unsupported argument";
        case SCONV_ERR_LAUNCH: return "kernel launch failed";
    }
    return "unknown status";
}

sconv_status sconv_fused(const void *x, int64_t x_row_stride, int T, int C, const void *weight,
                         int64_t w_stride_c, int64_t w_stride_k, int W, void *cache,
                         const int64_t cache_strides[4], int64_t num_blocks, int H, int N, int D,
                         const int64_t *positions, const int32_t *seq_idx,
                         const int64_t *slot_mapping, const int32_t *query_start,
                         const int32_t *block_table, int64_t bt_row_stride, int num_reqs,
                         int max_blocks, int off_s, int ws, sconv_act act, int use_residual,
                         sconv_dtype dt, void *out, int64_t out_row_stride, int32_t *err_flag,
                         cudaStream_t stream) {
    if (T < 0) return SCONV_ERR_INVALID;
    if (T == 0) return SCONV_OK;
    if (!seq_idx || !query_start) return SCONV_ERR_INVALID;
    FusedArgs a;
    bool vec = false;
    const sconv_status st = check_fused(
        x, x_row_stride, T, C, weight, w_stride_c, w_stride_k, W, cache, cache_strides,
        num_blocks, H, N, D, positions, slot_mapping, block_table, bt_row_stride, num_reqs,
        max_blocks, off_s, ws, act, use_residual, dt, out, out_row_stride, err_flag, a, vec);
    if (st != SCONV_OK) return st;
    a.seq_idx = seq_idx;
    a.qstart = query_start;
    return sconv::launch_fused(a, dt == SCONV_BF16, vec, false, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_fused_streams(const sconv_stream_desc *streams, int n_streams, int T, int W,
                                 void *cache, const int64_t cache_strides[4], int64_t num_blocks,
                                 int H, int N, int D, const int64_t *positions,
                                 const int32_t *seq_idx, const int64_t *slot_mapping,
                                 const int32_t *query_start, const int32_t *block_table,
                                 int64_t bt_row_stride, int num_reqs, int max_blocks,
                                 sconv_dtype dt, int32_t *err_flag, cudaStream_t stream) {
    if (T < 0 || n_streams < 1 || !streams) return SCONV_ERR_INVALID;
    if (n_streams > SCONV_MAX_STREAMS) return SCONV_ERR_UNSUPPORTED;
    if (T == 0) return SCONV_OK;
    if (!seq_idx || !query_start) return SCONV_ERR_INVALID;
    FusedArgs a[SCONV_MAX_STREAMS];
    bool vec_all = true;
    const int64_t e = elem_size(dt);
    for (int i = 0; i < n_streams; ++i) {
        const sconv_stream_desc &d = streams[i];
        bool vec = false;
        const sconv_status st = check_fused(
            d.x, d.x_row_stride, T, H * d.ws, d.weight, d.w_stride_c, d.w_stride_k, W, cache,
            cache_strides, num_blocks, H, N, D, positions, slot_mapping, block_table,
            bt_row_stride, num_reqs, max_blocks, d.off_s, d.ws, d.act, d.use_residual, dt, d.out,
            d.out_row_stride, err_flag, a[i], vec);
        if (st != SCONV_OK) return st;
        a[i].seq_idx = seq_idx;
        a[i].qstart = query_start;
        vec_all = vec_all && vec;
        const int64_t out_bytes =
            ((static_cast<int64_t>(T) - 1) * d.out_row_stride + H * d.ws) * e;
        for (int j = 0; j < i; ++j) {
            const sconv_stream_desc &o = streams[j];
            // lane ranges disjoint
            if (d.off_s < o.off_s + o.ws && o.off_s < d.off_s + d.ws) return SCONV_ERR_INVALID;
            const int64_t o_out = ((static_cast<int64_t>(T) - 1) * o.out_row_stride + H * o.ws) * e;
            const int64_t o_x = ((static_cast<int64_t>(T) - 1) * o.x_row_stride + H * o.ws) * e;
            const int64_t d_x = ((static_cast<int64_t>(T) - 1) * d.x_row_stride + H * d.ws) * e;
            if (overlaps(d.out, out_bytes, o.out, o_out) || overlaps(d.out, out_bytes, o.x, o_x) ||
                overlaps(o.out, o_out, d.x, d_x))
                return SCONV_ERR_INVALID;
        }
    }
    return sconv::launch_fused_streams(a, n_streams, dt == SCONV_BF16, vec_all, stream) ==
                   cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

}  // extern "C"

namespace {
// Shared checks of sconv_fused_taps and sconv_fused_taps_next (T > 0).
sconv_status check_taps_call(const sconv_stream_desc *streams, int n_streams, int T, int W,
                             void *cache, const int64_t cache_strides[4], int64_t num_blocks,
                             int H, int N, int D, const int64_t *slot_mapping, const int64_t *taps,
                             sconv_dtype dt, int32_t *err_flag, FusedArgs *a, bool &vec_all) {
    if (W > 1 && !taps) return SCONV_ERR_INVALID;
    vec_all = true;
    const int64_t e = elem_size(dt);
    const int64_t taps_bytes = static_cast<int64_t>(T) * (W > 1 ? W - 1 : 0) * 8;
    for (int i = 0; i < n_streams; ++i) {
        const sconv_stream_desc &d = streams[i];
        bool vec = false;
        const sconv_status st = check_fused(
            d.x, d.x_row_stride, T, H * d.ws, d.weight, d.w_stride_c, d.w_stride_k, W, cache,
            cache_strides, num_blocks, H, N, D, nullptr, slot_mapping, nullptr, 0, 0, 0,
            d.off_s, d.ws, d.act, d.use_residual, dt, d.out, d.out_row_stride, err_flag, a[i],
            vec, false);
        if (st != SCONV_OK) return st;
        a[i].taps = taps;
        vec_all = vec_all && vec;
        const int64_t out_bytes =
            ((static_cast<int64_t>(T) - 1) * d.out_row_stride + H * d.ws) * e;
        if (taps_bytes && overlaps(d.out, out_bytes, taps, taps_bytes)) return SCONV_ERR_INVALID;
        for (int j = 0; j < i; ++j) {
            const sconv_stream_desc &o = streams[j];
            if (d.off_s < o.off_s + o.ws && o.off_s < d.off_s + d.ws) return SCONV_ERR_INVALID;
            const int64_t o_out = ((static_cast<int64_t>(T) - 1) * o.out_row_stride + H * o.ws) * e;
            const int64_t o_x = ((static_cast<int64_t>(T) - 1) * o.x_row_stride + H * o.ws) * e;
            const int64_t d_x = ((static_cast<int64_t>(T) - 1) * d.x_row_stride + H * d.ws) * e;
            if (overlaps(d.out, out_bytes, o.out, o_out) || overlaps(d.out, out_bytes, o.x, o_x) ||
                overlaps(o.out, o_out, d.x, d_x))
                return SCONV_ERR_INVALID;
        }
    }
    return SCONV_OK;
}
}  // namespace

extern "C" {

sconv_status sconv_fused_taps(const sconv_stream_desc *streams, int n_streams, int T, int W,
                              void *cache, const int64_t cache_strides[4], int64_t num_blocks,
                              int H, int N, int D, const int64_t *slot_mapping,
                              const int64_t *taps, int metadata_ready, sconv_dtype dt,
                              int32_t *err_flag, cudaStream_t stream) {
    if (T < 0 || n_streams < 1 || !streams) return SCONV_ERR_INVALID;
    if (n_streams > SCONV_MAX_STREAMS) return SCONV_ERR_UNSUPPORTED;
    if (T == 0) return SCONV_OK;
    FusedArgs a[SCONV_MAX_STREAMS];
    bool vec_all = true;
    const sconv_status st = check_taps_call(streams, n_streams, T, W, cache, cache_strides,
                                            num_blocks, H, N, D, slot_mapping, taps, dt, err_flag,
                                            a, vec_all);
    if (st != SCONV_OK) return st;
    return sconv::launch_fused_taps(a, n_streams, dt == SCONV_BF16, vec_all,
                                    metadata_ready != 0, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_update(const void *x, int64_t x_row_stride, int B, int C, const void *weight,
                          int64_t w_stride_c, int64_t w_stride_k, int W, void *cache,
                          const int64_t cache_strides[4], int64_t num_blocks, int H, int N,
                          int D, const int64_t *positions, const int64_t *slot_mapping,
                          const int32_t *block_table, int64_t bt_row_stride, int max_blocks,
                          int off_s, int ws, sconv_act act, int use_residual, sconv_dtype dt,
                          void *out, int64_t out_row_stride, int32_t *err_flag,
                          cudaStream_t stream) {
    if (B < 0) return SCONV_ERR_INVALID;
    if (B == 0) return SCONV_OK;
    FusedArgs a;
    bool vec = false;
    const sconv_status st = check_fused(
        x, x_row_stride, B, C, weight, w_stride_c, w_stride_k, W, cache, cache_strides,
        num_blocks, H, N, D, positions, slot_mapping, block_table, bt_row_stride, B, max_blocks,
        off_s, ws, act, use_residual, dt, out, out_row_stride, err_flag, a, vec);
    if (st != SCONV_OK) return st;
    return sconv::launch_fused(a, dt == SCONV_BF16, vec, true, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_extract_windows(const void *src, int64_t seq_len, int conv_dim,
                                   int64_t src_stride_s, int64_t src_stride_c,
                                   const int32_t *abs_positions, const int32_t *real_count,
                                   int max_count, void *out, int64_t out_slot_stride, int d_conv,
                                   sconv_dtype dt, cudaStream_t stream) {
    if (dt != SCONV_F32 && dt != SCONV_BF16) return SCONV_ERR_UNSUPPORTED;
    if (max_count < 0 || conv_dim < 1 || seq_len < 0 || d_conv < 1) return SCONV_ERR_INVALID;
    if (d_conv > SCONV_MAX_DCONV) return SCONV_ERR_UNSUPPORTED;
    if (max_count == 0) return SCONV_OK;
    if (!src || !abs_positions || !real_count || !out) return SCONV_ERR_INVALID;
    if (src_stride_c != 1 || src_stride_s < conv_dim) return SCONV_ERR_INVALID;
    if (out_slot_stride < static_cast<int64_t>(conv_dim) * d_conv) return SCONV_ERR_INVALID;
    const int64_t e = elem_size(dt);
    const int64_t out_bytes =
        ((static_cast<int64_t>(max_count) - 1) * out_slot_stride +
         static_cast<int64_t>(conv_dim) * d_conv) * e;
    const int64_t src_bytes =
        seq_len > 0 ? ((seq_len - 1) * src_stride_s + conv_dim) * e : 0;
    if (src_bytes > 0 && overlaps(out, out_bytes, src, src_bytes)) return SCONV_ERR_INVALID;

    const int64_t V = 16 / e;
    const bool vec = aligned16(src) && aligned16(out) && src_stride_s % V == 0 &&
                     conv_dim % V == 0 && out_slot_stride % V == 0;
    sconv::ExtractArgs a;
    a.src = src;
    a.seq_len = seq_len;
    a.conv_dim = conv_dim;
    a.src_ss = src_stride_s;
    a.abs_pos = abs_positions;
    a.real_count = real_count;
    a.max_count = max_count;
    a.out = out;
    a.out_ss = out_slot_stride;
    a.d_conv = d_conv;
    return sconv::launch_extract(a, dt == SCONV_BF16, vec, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_scatter_intermediate_ssm(const void *states, int64_t num_chunks,
                                            int64_t state_flat, int64_t states_row_stride,
                                            const int64_t *chunk_indices,
                                            const int32_t *real_count, int max_count, void *out,
                                            int64_t out_row_stride, sconv_dtype dt,
                                            int32_t *err_flag, cudaStream_t stream) {
    if (dt != SCONV_F32 && dt != SCONV_BF16) return SCONV_ERR_UNSUPPORTED;
    if (max_count < 0 || num_chunks < 0 || state_flat < 1) return SCONV_ERR_INVALID;
    if (max_count > 65535) return SCONV_ERR_UNSUPPORTED;  // one grid row per slot
    if (max_count == 0) return SCONV_OK;
    if (!states || !chunk_indices || !real_count || !out) return SCONV_ERR_INVALID;
    if (states_row_stride < state_flat || out_row_stride < state_flat) return SCONV_ERR_INVALID;
    const int64_t e = elem_size(dt);
    const int64_t out_bytes = ((max_count - 1) * out_row_stride + state_flat) * e;
    const int64_t st_bytes = num_chunks > 0 ? ((num_chunks - 1) * states_row_stride + state_flat) * e : 0;
    if (st_bytes > 0 && overlaps(out, out_bytes, states, st_bytes)) return SCONV_ERR_INVALID;
    const bool vec = aligned16(states) && aligned16(out) && (state_flat * e) % 16 == 0 &&
                     (states_row_stride * e) % 16 == 0 && (out_row_stride * e) % 16 == 0;
    sconv::SsmArgs a;
    a.states = states;
    a.num_chunks = num_chunks;
    a.state_flat = state_flat;
    a.states_rs = states_row_stride;
    a.idx = chunk_indices;
    a.real_count = real_count;
    a.max_count = max_count;
    a.out = out;
    a.out_rs = out_row_stride;
    a.err = err_flag;
    return sconv::launch_scatter_ssm(a, static_cast<int>(e), vec, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_extract_windows_paged(const void *cache, const int64_t cache_strides[4],
                                         int64_t num_blocks, int H, int N, int D, int off_s,
                                         int ws, const int32_t *block_table,
                                         int64_t bt_row_stride, int num_reqs, int max_blocks,
                                         const int32_t *request, const int32_t *abs_positions,
                                         const int32_t *real_count, int max_count, void *out,
                                         int64_t out_slot_stride, int d_conv, sconv_dtype dt,
                                         int32_t *err_flag, cudaStream_t stream) {
    if (dt != SCONV_F32 && dt != SCONV_BF16) return SCONV_ERR_UNSUPPORTED;
    if (max_count < 0 || d_conv < 1) return SCONV_ERR_INVALID;
    if (d_conv > SCONV_MAX_DCONV) return SCONV_ERR_UNSUPPORTED;
    if (max_count == 0) return SCONV_OK;
    if (H < 1 || N < 1 || D < 1 || ws < 1 || off_s < 0 || static_cast<int64_t>(off_s) + ws > D)
        return SCONV_ERR_INVALID;
    if (num_blocks < 1 || num_reqs < 1 || max_blocks < 1 || bt_row_stride < max_blocks)
        return SCONV_ERR_INVALID;
    if (!cache || !cache_strides || !block_table || !request || !abs_positions || !real_count ||
        !out)
        return SCONV_ERR_INVALID;
    if (cache_strides[3] != 1 || cache_strides[0] < 1 || cache_strides[1] < 1 ||
        cache_strides[2] < 1)
        return SCONV_ERR_INVALID;
    const int64_t C = static_cast<int64_t>(H) * ws;
    if (out_slot_stride < C * d_conv) return SCONV_ERR_INVALID;
    const int64_t e = elem_size(dt);
    const int64_t out_bytes = ((max_count - 1) * out_slot_stride + C * d_conv) * e;
    const int64_t cache_bytes = ((num_blocks - 1) * cache_strides[0] +
                                 static_cast<int64_t>(H - 1) * cache_strides[1] +
                                 static_cast<int64_t>(N - 1) * cache_strides[2] + D) * e;
    if (overlaps(out, out_bytes, cache, cache_bytes)) return SCONV_ERR_INVALID;
    const int64_t V = 16 / e;
    const bool vec = aligned16(cache) && aligned16(out) && cache_strides[0] % V == 0 &&
                     cache_strides[1] % V == 0 && cache_strides[2] % V == 0 && off_s % V == 0 &&
                     ws % V == 0 && out_slot_stride % V == 0;
    sconv::PagedExtractArgs a;
    a.cache = cache;
    a.cs0 = cache_strides[0];
    a.cs1 = cache_strides[1];
    a.cs2 = cache_strides[2];
    a.num_blocks = num_blocks;
    a.H = H;
    a.N = N;
    a.off_s = off_s;
    a.ws = ws;
    a.bt = block_table;
    a.bt_rs = bt_row_stride;
    a.num_reqs = num_reqs;
    a.max_blocks = max_blocks;
    a.request = request;
    a.abs_pos = abs_positions;
    a.real_count = real_count;
    a.max_count = max_count;
    a.out = out;
    a.out_ss = out_slot_stride;
    a.d_conv = d_conv;
    a.err = err_flag;
    return sconv::launch_extract_paged(a, dt == SCONV_BF16, vec, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_causal_conv1d_fwd(
    void *x, int64_t x_stride_t, int64_t x_stride_c, int total_tokens, int dim,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W, const void *bias,
    void *conv_states, int64_t s_stride_line, int64_t s_stride_c, int64_t s_stride_k,
    int state_len, int num_lines, const int32_t *query_start_loc, int batch,
    const int32_t *cache_indices, const uint8_t *has_initial_state, sconv_act act,
    int pad_slot_id, void *out, sconv_dtype dt, int32_t *err_flag, cudaStream_t stream) {
    if (batch < 0) return SCONV_ERR_INVALID;
    sconv::DenseArgs a;
    bool vec = false;
    const sconv_status st = check_dense(
        x, x_stride_t, x_stride_c, total_tokens, dim, weight, w_stride_c, w_stride_k, W, bias,
        conv_states, s_stride_line, s_stride_c, s_stride_k, state_len, num_lines, act, out, dt,
        a, vec);
    if (st != SCONV_OK) return st;
    if (batch == 0) return SCONV_OK;
    if (!query_start_loc) return SCONV_ERR_INVALID;
    // grids: (sequence, column) blocks, or one warp per (sequence, channel)
    if (static_cast<int64_t>(batch) * dim / 8 + 1 > INT32_MAX) return SCONV_ERR_UNSUPPORTED;
    a.qsl = query_start_loc;
    a.batch = batch;
    a.lines = cache_indices;
    a.init = has_initial_state;
    a.pad = pad_slot_id;
    a.err = err_flag;
    return sconv::launch_dense_fwd(a, dt == SCONV_BF16, vec, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_causal_conv1d_update(
    void *x, int64_t x_stride_b, int64_t x_stride_c, int batch, int dim,
    const void *weight, int64_t w_stride_c, int64_t w_stride_k, int W, const void *bias,
    void *conv_state, int64_t s_stride_line, int64_t s_stride_c, int64_t s_stride_k,
    int state_len, int num_lines, const int32_t *cache_seqlens,
    const int32_t *conv_state_indices, sconv_act act, int pad_slot_id, void *out,
    sconv_dtype dt, int32_t *err_flag, cudaStream_t stream) {
    if (batch < 0 || !conv_state) return SCONV_ERR_INVALID;
    sconv::DenseArgs a;
    bool vec = false;
    const sconv_status st = check_dense(
        x, x_stride_b, x_stride_c, batch, dim, weight, w_stride_c, w_stride_k, W, bias,
        conv_state, s_stride_line, s_stride_c, s_stride_k, state_len, num_lines, act, out, dt,
        a, vec);
    if (st != SCONV_OK) return st;
    if (batch == 0) return SCONV_OK;
    a.batch = batch;
    a.lines = conv_state_indices;
    a.seqlens = cache_seqlens;
    a.pad = pad_slot_id;
    a.err = err_flag;
    return sconv::launch_dense_update(a, dt == SCONV_BF16, vec, stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

namespace {
sconv_status seq_metadata(const int32_t *query_start_loc, int num_reqs, int num_actual_tokens,
                          int num_padded_tokens, int32_t *seq_idx_out, int64_t seq_idx_cap,
                          int32_t *query_start_out, int64_t query_start_cap, bool ahead,
                          cudaStream_t stream) {
    if (num_padded_tokens < 0) num_padded_tokens = num_actual_tokens;
    if (num_actual_tokens < 0 || num_reqs < 0) return SCONV_ERR_INVALID;
    if (num_padded_tokens < num_actual_tokens) return SCONV_ERR_INVALID;
    if (num_padded_tokens > seq_idx_cap || num_padded_tokens > query_start_cap)
        return SCONV_ERR_INVALID;
    if (num_actual_tokens > 0 && num_reqs < 1) return SCONV_ERR_INVALID;
    if (num_padded_tokens == 0) return SCONV_OK;
    if (!query_start_loc || !seq_idx_out || !query_start_out) return SCONV_ERR_INVALID;
    return sconv::launch_seq_metadata(query_start_loc, num_reqs, num_actual_tokens,
                                      num_padded_tokens, seq_idx_out, query_start_out, ahead,
                                      stream) == cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}
}  // namespace

namespace {
// Checks of a tap resolution; on SCONV_OK fills `a`, and `empty` says there
// is nothing to write.
sconv_status resolve_args(const int32_t *qsl, int num_reqs, int num_actual, int num_padded,
                          const int64_t *positions, const int64_t *slot_mapping,
                          const int32_t *block_table, int64_t bt_rs, int max_blocks,
                          int64_t num_blocks, int N, int W, int32_t *seq_idx_out,
                          int64_t seq_idx_cap, int32_t *query_start_out,
                          int64_t query_start_cap, int64_t *taps_out, int64_t taps_cap,
                          sconv::TapResolveArgs &a, bool &empty) {
    empty = true;
    if (num_padded < 0) num_padded = num_actual;
    if (num_actual < 0 || num_reqs < 0 || num_padded < num_actual) return SCONV_ERR_INVALID;
    if (W < 1) return SCONV_ERR_INVALID;
    if (W > SCONV_MAX_W) return SCONV_ERR_UNSUPPORTED;
    if (N < 1 || num_blocks < 1 || max_blocks < 1 || bt_rs < max_blocks) return SCONV_ERR_INVALID;
    if (num_actual > 0 && num_reqs < 1) return SCONV_ERR_INVALID;
    if ((seq_idx_out && num_padded > seq_idx_cap) ||
        (query_start_out && num_padded > query_start_cap))
        return SCONV_ERR_INVALID;
    if (static_cast<int64_t>(num_padded) * (W - 1) > taps_cap) return SCONV_ERR_INVALID;
    if (num_padded == 0) return SCONV_OK;
    if ((W > 1 && !taps_out) || (num_actual > 0 && (!positions || !slot_mapping || !block_table)))
        return SCONV_ERR_INVALID;
    if (W == 1 && !seq_idx_out && !query_start_out) return SCONV_OK;  // nothing to write
    a = sconv::TapResolveArgs{};
    a.qsl = qsl;
    a.num_reqs = num_reqs;
    a.num_actual = num_actual;
    a.num_padded = num_padded;
    a.positions = positions;
    a.slot = slot_mapping;
    a.bt = block_table;
    a.bt_rs = bt_rs;
    a.max_blocks = max_blocks;
    a.num_blocks = num_blocks;
    a.N = N;
    a.W = W;
    a.seq_idx = seq_idx_out;
    a.qstart = query_start_out;
    a.taps = taps_out;
    empty = false;
    return SCONV_OK;
}

sconv_status seq_metadata_taps(const int32_t *qsl, int num_reqs, int num_actual,
                               int num_padded, const int64_t *positions,
                               const int64_t *slot_mapping, const int32_t *block_table,
                               int64_t bt_rs, int max_blocks, int64_t num_blocks, int N, int W,
                               int32_t *seq_idx_out, int64_t seq_idx_cap,
                               int32_t *query_start_out, int64_t query_start_cap,
                               int64_t *taps_out, int64_t taps_cap, bool ahead,
                               cudaStream_t stream) {
    sconv::TapResolveArgs a;
    bool empty = true;
    const sconv_status st = resolve_args(qsl, num_reqs, num_actual, num_padded, positions,
                                         slot_mapping, block_table, bt_rs, max_blocks, num_blocks,
                                         N, W, seq_idx_out, seq_idx_cap, query_start_out,
                                         query_start_cap, taps_out, taps_cap, a, empty);
    if (st != SCONV_OK || empty) return st;
    return sconv::launch_seq_metadata_taps(a, ahead, stream) == cudaSuccess ? SCONV_OK
                                                                            : SCONV_ERR_LAUNCH;
}
}  // namespace

sconv_status sconv_fused_taps_next(const sconv_stream_desc *streams, int n_streams, int T, int W,
                                   void *cache, const int64_t cache_strides[4],
                                   int64_t num_blocks, int H, int N, int D,
                                   const int64_t *slot_mapping, const int64_t *taps,
                                   sconv_dtype dt, int32_t *err_flag,
                                   const sconv_taps_build *next, cudaStream_t stream) {
    if (T < 0 || n_streams < 1 || !streams || !next) return SCONV_ERR_INVALID;
    if (n_streams > SCONV_MAX_STREAMS) return SCONV_ERR_UNSUPPORTED;
    sconv::TapResolveArgs nx;
    bool empty = true;
    sconv_status st = resolve_args(
        next->query_start_loc, next->num_reqs, next->num_actual_tokens,
        next->num_padded_tokens, next->positions, next->slot_mapping, next->block_table,
        next->bt_row_stride, next->max_blocks, num_blocks, N, W, next->seq_idx_out,
        next->seq_idx_cap, next->query_start_out, next->query_start_cap, next->taps_out,
        next->taps_cap, nx, empty);
    if (st != SCONV_OK) return st;
    if (T == 0) {
        if (empty) return SCONV_OK;
        return sconv::launch_seq_metadata_taps(nx, true, stream) == cudaSuccess
                   ? SCONV_OK
                   : SCONV_ERR_LAUNCH;
    }
    FusedArgs a[SCONV_MAX_STREAMS];
    bool vec_all = true;
    st = check_taps_call(streams, n_streams, T, W, cache, cache_strides, num_blocks, H, N, D,
                         slot_mapping, taps, dt, err_flag, a, vec_all);
    if (st != SCONV_OK) return st;
    if (!empty && next->taps_out && W > 1) {
        const int64_t nb = static_cast<int64_t>(nx.num_padded) * (W - 1) * 8;
        const int64_t tb = static_cast<int64_t>(T) * (W - 1) * 8;
        if (overlaps(next->taps_out, nb, taps, tb)) return SCONV_ERR_INVALID;
        const int64_t e = elem_size(dt);
        for (int i = 0; i < n_streams; ++i) {
            const sconv_stream_desc &d = streams[i];
            const int64_t out_bytes =
                ((static_cast<int64_t>(T) - 1) * d.out_row_stride + H * d.ws) * e;
            if (overlaps(next->taps_out, nb, d.out, out_bytes)) return SCONV_ERR_INVALID;
        }
    }
    if (empty)
        return sconv::launch_fused_taps(a, n_streams, dt == SCONV_BF16, vec_all, false, stream) ==
                       cudaSuccess
                   ? SCONV_OK
                   : SCONV_ERR_LAUNCH;
    return sconv::launch_fused_taps_next(a, n_streams, dt == SCONV_BF16, vec_all, nx, stream) ==
                   cudaSuccess
               ? SCONV_OK
               : SCONV_ERR_LAUNCH;
}

sconv_status sconv_seq_metadata_taps(const int32_t *query_start_loc, int num_reqs,
                                     int num_actual_tokens, int num_padded_tokens,
                                     const int64_t *positions, const int64_t *slot_mapping,
                                     const int32_t *block_table, int64_t bt_row_stride,
                                     int max_blocks, int64_t num_blocks, int N, int W,
                                     int32_t *seq_idx_out, int64_t seq_idx_cap,
                                     int32_t *query_start_out, int64_t query_start_cap,
                                     int64_t *taps_out, int64_t taps_cap, cudaStream_t stream) {
    return seq_metadata_taps(query_start_loc, num_reqs, num_actual_tokens, num_padded_tokens,
                             positions, slot_mapping, block_table, bt_row_stride, max_blocks,
                             num_blocks, N, W, seq_idx_out, seq_idx_cap, query_start_out,
                             query_start_cap, taps_out, taps_cap, false, stream);
}

sconv_status sconv_seq_metadata_taps_ahead(
    const int32_t *query_start_loc, int num_reqs, int num_actual_tokens, int num_padded_tokens,
    const int64_t *positions, const int64_t *slot_mapping, const int32_t *block_table,
    int64_t bt_row_stride, int max_blocks, int64_t num_blocks, int N, int W,
    int32_t *seq_idx_out, int64_t seq_idx_cap, int32_t *query_start_out,
    int64_t query_start_cap, int64_t *taps_out, int64_t taps_cap, cudaStream_t stream) {
    return seq_metadata_taps(query_start_loc, num_reqs, num_actual_tokens, num_padded_tokens,
                             positions, slot_mapping, block_table, bt_row_stride, max_blocks,
                             num_blocks, N, W, seq_idx_out, seq_idx_cap, query_start_out,
                             query_start_cap, taps_out, taps_cap, true, stream);
}

sconv_status sconv_seq_metadata(const int32_t *query_start_loc, int num_reqs,
                                int num_actual_tokens, int num_padded_tokens,
                                int32_t *seq_idx_out, int64_t seq_idx_cap,
                                int32_t *query_start_out, int64_t query_start_cap,
                                cudaStream_t stream) {
    return seq_metadata(query_start_loc, num_reqs, num_actual_tokens, num_padded_tokens,
                        seq_idx_out, seq_idx_cap, query_start_out, query_start_cap, false,
                        stream);
}

sconv_status sconv_seq_metadata_ahead(const int32_t *query_start_loc, int num_reqs,
                                      int num_actual_tokens, int num_padded_tokens,
                                      int32_t *seq_idx_out, int64_t seq_idx_cap,
                                      int32_t *query_start_out, int64_t query_start_cap,
                                      cudaStream_t stream) {
    return seq_metadata(query_start_loc, num_reqs, num_actual_tokens, num_padded_tokens,
                        seq_idx_out, seq_idx_cap, query_start_out, query_start_cap, true,
                        stream);
}

}  // extern "C"
