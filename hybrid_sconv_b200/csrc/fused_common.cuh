// fused_common.cuh -- per-token helpers shared by the fused kernels
// (token, strip and TMA forms), so that every form resolves taps, checks
// indices and addresses the cache in exactly the same way.
#pragma once

#include "common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

struct Tok {
    int64_t pos, slot;
    int req, q0;
};

template <bool ONE>
__device__ __forceinline__ Tok load_tok(const FusedArgs &a, int t) {
    Tok k;
    k.pos = __ldg(a.positions + t);
    k.slot = __ldg(a.slot + t);
    if (ONE) {
        k.req = t;
        k.q0 = t;
    } else {
        k.req = __ldg(a.seq_idx + t);
        k.q0 = __ldg(a.qstart + t);
    }
    return k;
}

// Block and offset of a non-negative position or slot.
__device__ __forceinline__ void split_n(const FusedArgs &a, int64_t v, bool fast32, int64_t &blk,
                                        int64_t &off) {
    if (fast32) {
        const uint32_t q = a.divN.div(static_cast<uint32_t>(v));
        blk = q;
        off = static_cast<int64_t>(static_cast<uint32_t>(v) - q * a.divN.d);
    } else {
        blk = v / a.N;
        off = v - blk * a.N;
    }
}

// Range checks of a non-PAD token's own indices (SCONV_EFLAG_* bits).
template <bool ONE>
__device__ __forceinline__ unsigned check_tok(const FusedArgs &a, const Tok &k, int t) {
    unsigned bad = 0;
    if (k.slot < 0 || k.slot >= a.num_blocks * a.N) bad |= SCONV_EFLAG_SLOT;
    if (!ONE) {
        if (k.req < 0 || k.req >= a.num_reqs) bad |= SCONV_EFLAG_REQUEST;
        if (k.q0 < 0 || k.q0 > t) bad |= SCONV_EFLAG_QUERY_START;
    }
    if (k.pos < 0) bad |= SCONV_EFLAG_POSITION;
    return bad;
}

// The taps of the thread's VEC channels as floats, indexed by lag d
// (wr[d] multiplies position pos - d, i.e. weight column W-1-d).
template <typename E, int VEC, int MAXW>
__device__ __forceinline__ void load_weights(const FusedArgs &a, int c, float (&wr)[MAXW][VEC]) {
    const E *w = static_cast<const E *>(a.w);
    if constexpr (VEC * sizeof(E) == 16) {
        if (a.w_vec) {  // dense [C, W] with W == MAXW: VEC*MAXW contiguous elements
            union {
                uint4 u[MAXW];
                E e[VEC * MAXW];
            } raw;
            const uint4 *p = reinterpret_cast<const uint4 *>(w + static_cast<int64_t>(c) * MAXW);
#pragma unroll
            for (int q = 0; q < MAXW; ++q) raw.u[q] = __ldg(p + q);
#pragma unroll
            for (int v = 0; v < VEC; ++v)
#pragma unroll
                for (int d = 0; d < MAXW; ++d) {
                    if constexpr (sizeof(E) == 2)
                        wr[d][v] = __uint_as_float(
                            static_cast<uint32_t>(reinterpret_cast<const unsigned short &>(
                                raw.e[v * MAXW + MAXW - 1 - d]))
                            << 16);
                    else
                        wr[d][v] = reinterpret_cast<const float &>(raw.e[v * MAXW + MAXW - 1 - d]);
                }
            return;
        }
    }
    const int W = a.W;
#pragma unroll
    for (int d = 0; d < MAXW; ++d)
#pragma unroll
        for (int v = 0; v < VEC; ++v)
            wr[d][v] = d < W ? load_weight(w + static_cast<int64_t>(c + v) * a.w_sc +
                                           static_cast<int64_t>(W - 1 - d) * a.w_sk)
                             : 0.f;
}

// Load one pre-forward tap (position src >= 0) of request `req` from the
// cache, or record why it cannot be read.
template <typename E, int VEC>
__device__ __forceinline__ unsigned load_cache_tap(const FusedArgs &a, int req, int64_t src,
                                                   int64_t lane, Pack<E, VEC> &tap) {
    int64_t lb, off;
    split_n(a, src, src < (1ll << 31), lb, off);
    if (lb >= a.max_blocks) return SCONV_EFLAG_LOGICAL;
    const int32_t b = __ldg(a.bt + static_cast<int64_t>(req) * a.bt_rs + lb);
    if (b < 0 || b >= a.num_blocks) return SCONV_EFLAG_BLOCK;
    tap.load_nc(static_cast<const E *>(a.cache) + static_cast<int64_t>(b) * a.cs0 + off * a.cs2 +
                lane);
    return 0;
}

}  // namespace
}  // namespace sconv
