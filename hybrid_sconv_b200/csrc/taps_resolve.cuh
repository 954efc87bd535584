// taps_resolve.cuh -- the per-step tap resolution of one block's tokens,
// shared by the standalone builder (sconv_seq_metadata_taps) and the fused
// step that builds the next step's table beside its own convolution
// (sconv_fused_taps_next).
//
// "vllm.models.inkling.nvidia.ops.sconv", module docstring: a tap in the
// current forward comes from x, an earlier one from the cache through
// block_table[req, src / N] at offset src % N, a tap before position 0 is
// zero.  The request and its first row come from a binary search of
// query_start_loc (the last request starting at or before the token), or
// are the token itself in the decode form.  Row t of the table holds, for
// lag d = 1..W-1, SCONV_TAP_X, SCONV_TAP_ZERO, the flat cache slot
// b*N + src % N, or -(bits << 8) at every lag when the token cannot be
// resolved.  A thread issues its W-1 block-table loads together, so the
// lookup is two dependent accesses (positions and query_start_loc, then the
// block table).
#pragma once

#include "common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

// Every thread of the block calls this (it may synchronise the block to
// stage query_start_loc in s_qsl): token t, thread tid of nthr.
template <bool DECODE, int MAXW>
__device__ __forceinline__ void resolve_block(const TapResolveArgs &a, int t, int tid, int nthr,
                                              int32_t *s_qsl) {
    const bool live = t < a.num_actual;
    int64_t pos = 0, slot = -1;
    if (live) {
        pos = __ldg(a.positions + t);
        slot = __ldg(a.slot + t);
    }
    if (!DECODE && a.staged) {
        for (int i = tid; i < a.num_reqs; i += nthr) s_qsl[i] = __ldg(a.qsl + i);
        __syncthreads();
    }
    if (t >= a.num_padded) return;
    int r = 0, q0 = 0;
    if (live) {
        if (DECODE) {
            r = t;
            q0 = t;
        } else {
            const int32_t *q = a.staged ? s_qsl : a.qsl;
            int lo = 0, hi = a.num_reqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (q[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            r = lo;
            q0 = q[lo];
        }
    }
    if (a.seq_idx) a.seq_idx[t] = r;
    if (a.qstart) a.qstart[t] = q0;

    int64_t e[MAXW];
#pragma unroll
    for (int d = 1; d < MAXW; ++d) e[d] = SCONV_TAP_ZERO;
    if (live && slot != -1) {
        unsigned flags = 0;
        if (r >= a.num_reqs) flags |= SCONV_EFLAG_REQUEST;
        if (q0 < 0 || q0 > t) flags |= SCONV_EFLAG_QUERY_START;
        if (pos < 0) flags |= SCONV_EFLAG_POSITION;
        if (!flags) {
            const int32_t *row = a.bt + static_cast<int64_t>(r) * a.bt_rs;
            int32_t blk[MAXW];
            int64_t off[MAXW];
            bool need[MAXW];
#pragma unroll
            for (int d = 1; d < MAXW; ++d) {  // issue every block-table load first
                need[d] = false;
                if (d >= a.W) continue;
                const int64_t src = pos - d;
                if (t - d >= q0) {
                    e[d] = SCONV_TAP_X;
                } else if (src >= 0) {
                    int64_t lb;
                    if (src < (1ll << 31)) {
                        const uint32_t q = a.divN.div(static_cast<uint32_t>(src));
                        lb = q;
                        off[d] = src - static_cast<int64_t>(q) * a.N;
                    } else {
                        lb = src / a.N;
                        off[d] = src - lb * a.N;
                    }
                    if (lb >= a.max_blocks) {
                        flags |= SCONV_EFLAG_LOGICAL;
                    } else {
                        blk[d] = __ldg(row + lb);
                        need[d] = true;
                    }
                }
            }
#pragma unroll
            for (int d = 1; d < MAXW; ++d) {
                if (!need[d]) continue;
                if (blk[d] < 0 || blk[d] >= a.num_blocks) flags |= SCONV_EFLAG_BLOCK;
                else e[d] = static_cast<int64_t>(blk[d]) * a.N + off[d];
            }
        }
        if (flags) {
#pragma unroll
            for (int d = 1; d < MAXW; ++d) e[d] = -static_cast<int64_t>(flags) * 256;
        }
    }
    int64_t *out = a.taps + static_cast<int64_t>(t) * (a.W - 1);
#pragma unroll
    for (int d = 1; d < MAXW; ++d)
        if (d < a.W) out[d - 1] = e[d];
}

// Shared memory of a block that runs resolve_block, and whether the
// offsets table is staged there.
inline void resolve_staging(TapResolveArgs &a, size_t &smem) {
    a.divN = FastDiv::make(static_cast<uint32_t>(a.N));
    a.staged = a.qsl != nullptr && a.num_reqs <= 4096 ? 1 : 0;
    smem = a.staged ? static_cast<size_t>(a.num_reqs) * sizeof(int32_t) : 0;
}

}  // namespace
}  // namespace sconv
