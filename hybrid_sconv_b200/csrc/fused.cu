// fused.cu -- one-launch cache insert + depthwise causal conv1d over the
// paged sliding-window cache ("vllm.models.inkling.nvidia.ops.sconv",
// module docstring and fused_sconv), for sm_100a.
//
// Per token t (position pos, request r, first x row of the request q0,
// slot s): a non-PAD token stores its x row into cache[s / N, h, s % N,
// off_s + j] and convolves, per channel, the W taps ending at pos.  Tap at
// lag d (position pos - d) is the x row t - d when that row is at or after
// q0, zero before position 0, else the cache element at block
// block_table[r, (pos - d) / N], offset (pos - d) % N.  out = act(conv) +
// (residual ? x : 0), fp32 accumulation from the oldest tap to the newest.
//
// A thread always owns one 16-byte channel pack (8 bf16 / 4 fp32, or one
// element for unaligned layouts), so every load and store of x, out and the
// cache is one 16-byte transaction and a warp covers 512 contiguous bytes of
// a row.  Two kernels share that layout:
//
//  * fused_token_kernel -- one token per thread.  Used when there are few
//    token-packs (decode, speculative decode): every load of a token
//    (metadata, x, block-table entries, cache taps) is issued as early as
//    its address is known, so a token costs three dependent DRAM round
//    trips (metadata -> block table -> cache) and nothing more.
//  * fused_strip_kernel -- a strip of L consecutive tokens per thread,
//    streamed through a register ring: the x row and metadata of token
//    t + PF are loaded while token t is computed, so loads are always in
//    flight and each x element is read from DRAM once (the W-1 halo rows
//    before the strip come from L2).  Used for the prefill shapes the tiled
//    form (fused_tma.cu) does not take: metadata or x not 16-byte aligned,
//    layouts without 16-byte channel packs, C below one tile row.
//
// The tap source (x, cache, zero) depends only on the token, so it is
// uniform across a warp.  The grid of either kernel is a function of T and
// C only, so every launch can be captured in a CUDA graph.  Both kernels
// start with griddepcontrol.wait (programmatic dependent launch), so they
// may be launched while the previous kernel in the stream drains.
#include "common.cuh"
#include "fused_common.cuh"
#include "sconv.h"
#include "taps_resolve.cuh"

namespace sconv {
namespace {

constexpr int kThreads = 256;

// Convolution, epilogue, output store and cache insert of one token.
// tap_of(d, use) returns the tap at lag d and sets `use` false for a tap
// that is zero (before position 0).
template <typename E, int VEC, int MAXW, typename TapFn>
__device__ __forceinline__ void conv_store_at(const FusedArgs &a, const float (&wr)[MAXW][VEC],
                                              TapFn tap_of, const Pack<E, VEC> &cur, E *out,
                                              E *ins) {
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
#pragma unroll
    for (int d = MAXW - 1; d >= 0; --d) {
        if (d >= a.W) continue;
        bool use = true;
        const Pack<E, VEC> p = tap_of(d, use);
        if (!use) continue;
        float f[VEC];
        p.to_float(f);
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wr[d][v], f[v], acc[v]);
    }
    float xc[VEC];
    cur.to_float(xc);
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        float y = acc[v];
        if (a.silu) y = silu<E>(y);
        if (a.resid) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
        acc[v] = y;
    }
    Pack<E, VEC> o;
    o.from_float(acc);
    o.store(out);
    cur.store(ins);
}

template <typename E, int VEC, int MAXW, typename TapFn>
__device__ __forceinline__ void conv_store(const FusedArgs &a, const float (&wr)[MAXW][VEC],
                                           TapFn tap_of, const Pack<E, VEC> &cur, int t, int c,
                                           int64_t slot, int64_t lane) {
    int64_t blk, off;
    split_n(a, slot, a.slots32 != 0, blk, off);
    conv_store_at<E, VEC, MAXW>(a, wr, tap_of, cur,
                                static_cast<E *>(a.out) + static_cast<int64_t>(t) * a.out_rs + c,
                                static_cast<E *>(a.cache) + blk * a.cs0 + off * a.cs2 + lane);
}

// Before the PDL wait, while the preceding kernel drains: pull token t's
// metadata, its x pack and (for a speculating launch) the pack's weights
// into L2 (a warp's lanes share t), then go one step further.  The token's
// metadata and block-table entries are read *speculatively* with L2-only
// loads (ld.global.cg, so no line enters L1) -- the preceding kernel may
// still be writing them -- and
// used only to choose which block-table lines and cache taps to prefetch
// into L2.  Every speculative index is range-checked before it forms an
// address.  After the wait the real loads run as usual; a stale value costs
// a useless prefetch, never a wrong result.
template <typename E, int MAXW, bool ONE, bool SPEC>
__device__ __forceinline__ void token_prefetch(const FusedArgs &a, int pack, int t, int vec) {
    if ((threadIdx.x & 31) == 0) {
        prefetch_l2(a.positions + t);
        prefetch_l2(a.slot + t);
        if (!ONE) {
            prefetch_l2(a.seq_idx + t);
            prefetch_l2(a.qstart + t);
        }
    }
    const int c = pack * vec;
    prefetch_l2(static_cast<const E *>(a.x) + static_cast<int64_t>(t) * a.x_rs + c);
    if (SPEC && a.w_vec) prefetch_l2(static_cast<const E *>(a.w) + static_cast<int64_t>(c) * a.W);
    if (!SPEC) return;

    const int64_t pos = __ldcg(a.positions + t);
    const int req = ONE ? t : __ldcg(a.seq_idx + t);
    const int q0 = ONE ? t : __ldcg(a.qstart + t);
    if (req < 0 || req >= a.num_reqs || pos < 0 || pos >= (1ll << 31)) return;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    const int32_t *bt_row = a.bt + static_cast<int64_t>(req) * a.bt_rs;
#pragma unroll
    for (int d = 1; d < MAXW; ++d) {
        if (d >= a.W || t - d >= q0 || pos - d < 0) continue;
        const uint32_t src = static_cast<uint32_t>(pos - d);
        const uint32_t lb = a.divN.div(src);
        if (lb >= static_cast<uint32_t>(a.max_blocks)) continue;
        const int32_t b = __ldcg(bt_row + lb);
        if (b < 0 || b >= a.num_blocks) continue;
        prefetch_l2(static_cast<const E *>(a.cache) + static_cast<int64_t>(b) * a.cs0 +
                    static_cast<int64_t>(src - lb * a.divN.d) * a.cs2 + lane);
    }
}

// One token-pack of the token kernel (after the PDL wait, in range).  PRE:
// the weights in wr were loaded before the wait; otherwise they are loaded
// here, after the token's first loads.
template <typename E, int VEC, int MAXW, bool ONE, bool PRE>
__device__ __forceinline__ void token_body(const FusedArgs &a, int pack, int t,
                                           float (&wr)[MAXW][VEC]) {
    using P = Pack<E, VEC>;
    const E *x = static_cast<const E *>(a.x);
    const int c = pack * VEC;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);

    const Tok k = load_tok<ONE>(a, t);
    P tap[MAXW];
    tap[0].load_nc(x + static_cast<int64_t>(t) * a.x_rs + c);
    if (!PRE) load_weights<E, VEC, MAXW>(a, c, wr);
    if (k.slot == -1) return;  // PAD row

    unsigned bad = check_tok<ONE>(a, k, t);
    bool use[MAXW];
    use[0] = true;
    if (!bad) {
#pragma unroll
        for (int d = 1; d < MAXW; ++d) {
            use[d] = false;
            if (d >= a.W) continue;
            const int64_t src = k.pos - d;
            if (t - d >= k.q0) {
                tap[d].load_nc(x + static_cast<int64_t>(t - d) * a.x_rs + c);
                use[d] = true;
            } else if (src >= 0) {
                bad |= load_cache_tap<E, VEC>(a, k.req, src, lane, tap[d]);
                use[d] = true;
            }
        }
    }
    if (bad) {
        if (a.err) atomicOr(a.err, static_cast<int>(bad));
        return;
    }
    conv_store<E, VEC, MAXW>(
        a, wr,
        [&](int d, bool &u) {
            u = use[d];
            return tap[d];
        },
        tap[0], t, c, k.slot, lane);
}

template <typename E, int VEC, int MAXW, bool ONE, bool SPEC>
__global__ void __launch_bounds__(kThreads) fused_token_kernel(const __grid_constant__ FusedArgs a) {
    const int pack = blockIdx.y * blockDim.x + threadIdx.x;
    const int t = blockIdx.x * blockDim.y + threadIdx.y;
    const bool in_range = pack < a.C / VEC && t < a.T;
    // Without speculation (a launch too large to sit beside its predecessor)
    // the weights are loaded into registers before the wait, which takes
    // their loads off the dependent chain (spec decode 6.10 -> 5.86 us); with
    // it they stay an L2 prefetch (loading them early made decode slower).
    float wr[MAXW][VEC];
    if (in_range) {
        token_prefetch<E, MAXW, ONE, SPEC>(a, pack, t, VEC);
        if (!SPEC) load_weights<E, VEC, MAXW>(a, pack * VEC, wr);
    }
    pdl_wait();
    pdl_trigger();
    if (in_range) token_body<E, VEC, MAXW, ONE, !SPEC>(a, pack, t, wr);
}

// Several conv streams of one layer (disjoint lane ranges of the same
// cache, the same tokens and metadata) in one launch: the grid's y blocks
// are the streams' channel blocks laid end to end.  Each block runs the
// token kernel's work for its stream, so the latency-bound chain (metadata
// -> block table -> cache) is paid once per launch for all streams.
struct StreamSet {
    FusedArgs s[SCONV_MAX_STREAMS];
    int n;
    int y0[SCONV_MAX_STREAMS + 1];  // first y block of each stream, y0[n] = total
};

// Runs f(args of stream si) with si a compile-time index in each branch, so
// the stream's fields are read from the parameter bank at fixed offsets (an
// index computed from blockIdx would turn every field read into an indexed
// load).
template <typename F>
__device__ __forceinline__ void with_stream(const StreamSet &m, int si, F f) {
    static_assert(SCONV_MAX_STREAMS == 4, "one branch per stream");
    switch (si) {
        case 0: f(m.s[0]); break;
        case 1: f(m.s[1]); break;
        case 2: f(m.s[2]); break;
        default: f(m.s[3]); break;
    }
}

template <typename E, int VEC, int MAXW, bool SPEC>
__device__ __forceinline__ void streams_body(const FusedArgs &a, int pack, int t) {
    const bool in_range = pack < a.C / VEC && t < a.T;
    float wr[MAXW][VEC];
    if (in_range) {
        token_prefetch<E, MAXW, false, SPEC>(a, pack, t, VEC);
        if (!SPEC) load_weights<E, VEC, MAXW>(a, pack * VEC, wr);
    }
    pdl_wait();
    pdl_trigger();
    if (in_range) token_body<E, VEC, MAXW, false, !SPEC>(a, pack, t, wr);
}

template <typename E, int VEC, int MAXW, bool SPEC>
__global__ void __launch_bounds__(kThreads) fused_streams_kernel(const __grid_constant__ StreamSet m) {
    int si = 0;
    while (si + 1 < m.n && static_cast<int>(blockIdx.y) >= m.y0[si + 1]) ++si;
    const int pack = (blockIdx.y - m.y0[si]) * blockDim.x + threadIdx.x;
    const int t = blockIdx.x * blockDim.y + threadIdx.y;
    with_stream(m, si, [&](const FusedArgs &a) { streams_body<E, VEC, MAXW, SPEC>(a, pack, t); });
}

// ---------------------------------------------------------------------------
// The fused step with resolved taps (sconv_fused_taps).  A token's tap
// sources come from one row of the table sconv_seq_metadata_taps built for
// the step: SCONV_TAP_X (x row t - d), SCONV_TAP_ZERO, a flat cache slot, or
// a failure code carrying SCONV_EFLAG_* bits.  The kernel reads no
// positions, request metadata or block table, so a token's taps are one
// dependent access after its slot and table row -- and with READY those are
// read before the PDL wait (the caller guarantees no kernel still running
// writes them), the x rows and cache taps are prefetched into L2 there, and
// after the wait only the x and cache loads remain.

template <int MAXW>
__device__ __forceinline__ void load_tap_row(const FusedArgs &a, int t, int64_t (&src)[MAXW]) {
    const int64_t *row = a.taps + static_cast<int64_t>(t) * (a.W - 1);
#pragma unroll
    for (int d = 1; d < MAXW; ++d) src[d] = d < a.W ? __ldg(row + d - 1) : SCONV_TAP_ZERO;
}

// SCONV_EFLAG_* bits of a non-PAD token: those its table row carries (an
// entry that is neither a valid slot, SCONV_TAP_X on a row of this call,
// SCONV_TAP_ZERO nor a failure code counts as SCONV_EFLAG_BLOCK), or, for a
// slot out of range, SCONV_EFLAG_SLOT with the row's request, query-start
// and position bits -- the bits sconv_fused reports for the same token.
template <int MAXW>
__device__ __forceinline__ unsigned tap_row_flags(const FusedArgs &a, int t, int64_t slot,
                                                  const int64_t (&src)[MAXW]) {
    const int64_t limit = a.num_blocks * a.N;
    unsigned f = 0;
#pragma unroll
    for (int d = 1; d < MAXW; ++d) {
        if (d >= a.W) continue;
        const int64_t e = src[d];
        if (e >= 0) {
            if (e >= limit) f |= SCONV_EFLAG_BLOCK;
        } else if (e == SCONV_TAP_X) {
            if (t - d < 0) f |= SCONV_EFLAG_QUERY_START;
        } else if (e != SCONV_TAP_ZERO) {
            const unsigned bits =
                e <= -256 ? static_cast<unsigned>((~static_cast<uint64_t>(e) + 1) >> 8) & 0x3fu
                          : 0u;
            f |= bits ? bits : SCONV_EFLAG_BLOCK;
        }
    }
    if (slot < 0 || slot >= limit)
        f = SCONV_EFLAG_SLOT |
            (f & (SCONV_EFLAG_REQUEST | SCONV_EFLAG_QUERY_START | SCONV_EFLAG_POSITION));
    return f;
}

// One token-pack of the resolved-tap form (pack, token t).  With READY the
// slot and table row are read before the PDL wait and the token's cache taps
// prefetched into L2 there; after the wait come the checks, the tap loads,
// the arithmetic and the two stores.  (Measured: this straight-line shape
// beats a form that carries precomputed addresses across the wait, 3.2 ->
// 2.4 us per decode launch.)  Without READY the table row is read
// speculatively before the wait with L2-only loads (the kernel that writes
// it may still be running), range-checked and used only to choose which
// cache taps to prefetch, and the token's slot_mapping line is prefetched;
// the real reads follow the wait.  (Measured on the decode chain without
// READY: the slot prefetch 2.91 -> 2.77 us per launch; also loading the
// taps at the speculative sources after the wait beside the real row, and
// keeping them where the two agree, 2.82: not kept.)
template <typename E, int VEC, int MAXW, bool READY>
__device__ __forceinline__ void taps_body(const FusedArgs &a, int pack, int t) {
    using P = Pack<E, VEC>;
    const bool in_range = pack < a.C / VEC && t < a.T;
    const int c = pack * VEC;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    const E *x = static_cast<const E *>(a.x);
    const E *cache = static_cast<const E *>(a.cache);

    float wr[MAXW][VEC];
    int64_t slot = -1;
    int64_t src[MAXW];
    if (in_range) {
        load_weights<E, VEC, MAXW>(a, c, wr);
        prefetch_l2(x + static_cast<int64_t>(t) * a.x_rs + c);
        if (READY) {
            slot = __ldg(a.slot + t);
            load_tap_row<MAXW>(a, t, src);
            const int64_t limit = a.num_blocks * a.N;
#pragma unroll
            for (int d = 1; d < MAXW; ++d) {
                if (src[d] >= 0 && src[d] < limit) {
                    int64_t blk, off;
                    split_n(a, src[d], a.slots32 != 0, blk, off);
                    prefetch_l2(cache + blk * a.cs0 + off * a.cs2 + lane);
                }
            }
        } else {
            prefetch_l2(a.slot + t);
            const int64_t *row = a.taps + static_cast<int64_t>(t) * (a.W - 1);
            const int64_t limit = a.num_blocks * a.N;
#pragma unroll
            for (int d = 1; d < MAXW; ++d) {
                if (d >= a.W) continue;
                const int64_t e = __ldcg(row + d - 1);
                if (e >= 0 && e < limit) {
                    int64_t blk, off;
                    split_n(a, e, a.slots32 != 0, blk, off);
                    prefetch_l2(cache + blk * a.cs0 + off * a.cs2 + lane);
                }
            }
        }
    }
    pdl_wait();
    pdl_trigger();
    if (!in_range) return;
    if (!READY) {
        slot = __ldg(a.slot + t);
        load_tap_row<MAXW>(a, t, src);
    }
    if (slot == -1) return;  // PAD row
    const unsigned bad = tap_row_flags<MAXW>(a, t, slot, src);
    if (bad) {
        if (a.err) atomicOr(a.err, static_cast<int>(bad));
        return;
    }
    P tap[MAXW];
    bool use[MAXW];
    tap[0].load_nc(x + static_cast<int64_t>(t) * a.x_rs + c);
    use[0] = true;
#pragma unroll
    for (int d = 1; d < MAXW; ++d) {
        use[d] = false;
        if (src[d] >= 0) {
            int64_t blk, off;
            split_n(a, src[d], a.slots32 != 0, blk, off);
            tap[d].load_nc(cache + blk * a.cs0 + off * a.cs2 + lane);
            use[d] = true;
        } else if (src[d] == SCONV_TAP_X) {
            tap[d].load_nc(x + static_cast<int64_t>(t - d) * a.x_rs + c);
            use[d] = true;
        }
    }
    conv_store<E, VEC, MAXW>(
        a, wr,
        [&](int d, bool &u) {
            u = use[d];
            return tap[d];
        },
        tap[0], t, c, slot, lane);
}

// One conv stream: the arguments are a plain kernel parameter.
template <typename E, int VEC, int MAXW, bool READY>
__global__ void __launch_bounds__(kThreads) fused_taps_kernel(const __grid_constant__ FusedArgs a) {
    taps_body<E, VEC, MAXW, READY>(a, blockIdx.y * blockDim.x + threadIdx.x,
                                   blockIdx.x * blockDim.y + threadIdx.y);
}

// Several streams of one layer in one launch: the grid's y blocks are the
// streams' channel blocks laid end to end.
template <typename E, int VEC, int MAXW, bool READY>
__global__ void __launch_bounds__(kThreads) fused_taps_streams_kernel(const __grid_constant__ StreamSet m) {
    int si = 0;
    while (si + 1 < m.n && static_cast<int>(blockIdx.y) >= m.y0[si + 1]) ++si;
    const int pack = (blockIdx.y - m.y0[si]) * blockDim.x + threadIdx.x;
    const int t = blockIdx.x * blockDim.y + threadIdx.y;
    with_stream(m, si, [&](const FusedArgs &a) { taps_body<E, VEC, MAXW, READY>(a, pack, t); });
}

// The fused step with the NEXT step's table built in the same launch
// (sconv_fused_taps_next): blocks with blockIdx.x < gx convolve this step
// (its table read after the wait, speculatively prefetched before it);
// blocks beyond build the next step's table from the next step's inputs,
// which no running kernel writes, so they neither wait nor hold back the
// launch of this grid's dependents (they signal at entry).  The next launch
// still waits for this whole grid before it reads that table.
template <bool DECODE_NEXT, int MAXW>
__device__ __forceinline__ void build_next(const TapResolveArgs &nx, int gx) {
    extern __shared__ int32_t s_qsl[];
    pdl_trigger();
    if (blockIdx.y != 0) return;  // one row of build blocks
    const int nthr = blockDim.x * blockDim.y;
    const int tid = threadIdx.y * blockDim.x + threadIdx.x;
    resolve_block<DECODE_NEXT, MAXW>(nx, (blockIdx.x - gx) * nthr + tid, tid, nthr, s_qsl);
}

constexpr int kNextThreads = 512;  // block size of the one-stream step at decode sizes

template <typename E, int VEC, int MAXW, bool DECODE_NEXT>
__global__ void __launch_bounds__(kNextThreads)
fused_taps_next_kernel(const __grid_constant__ FusedArgs a, const __grid_constant__ TapResolveArgs nx,
                       int gx) {
    if (static_cast<int>(blockIdx.x) >= gx) {
        build_next<DECODE_NEXT, MAXW>(nx, gx);
        return;
    }
    taps_body<E, VEC, MAXW, false>(a, blockIdx.y * blockDim.x + threadIdx.x,
                                   blockIdx.x * blockDim.y + threadIdx.y);
}

template <typename E, int VEC, int MAXW, bool DECODE_NEXT>
__global__ void __launch_bounds__(kThreads)
fused_taps_streams_next_kernel(const __grid_constant__ StreamSet m,
                               const __grid_constant__ TapResolveArgs nx, int gx) {
    if (static_cast<int>(blockIdx.x) >= gx) {
        build_next<DECODE_NEXT, MAXW>(nx, gx);
        return;
    }
    int si = 0;
    while (si + 1 < m.n && static_cast<int>(blockIdx.y) >= m.y0[si + 1]) ++si;
    const int pack = (blockIdx.y - m.y0[si]) * blockDim.x + threadIdx.x;
    const int t = blockIdx.x * blockDim.y + threadIdx.y;
    with_stream(m, si, [&](const FusedArgs &a) { taps_body<E, VEC, MAXW, false>(a, pack, t); });
}

// Ring of x rows: Q >= PF + MAXW slots, a power of two.
template <int PF, int MAXW>
struct Ring {
    static constexpr int need = PF + MAXW;
    static constexpr int Q = need <= 8 ? 8 : 16;
};

// Metadata of a 32-token chunk spread over a warp: lane l holds token
// chunk_start + l, and each token's fields are broadcast by shuffle when it
// is processed (one coalesced load per field per 32 tokens).
struct ChunkMeta {
    int64_t pos, slot;
    int req, q0;
};

__device__ __forceinline__ ChunkMeta load_chunk(const FusedArgs &a, int t, int t_end) {
    ChunkMeta m;
    if (t < t_end) {
        m.pos = __ldg(a.positions + t);
        m.slot = __ldg(a.slot + t);
        m.req = __ldg(a.seq_idx + t);
        m.q0 = __ldg(a.qstart + t);
    } else {
        m.pos = 0;
        m.slot = -1;
        m.req = 0;
        m.q0 = 0;
    }
    return m;
}

__device__ __forceinline__ Tok shfl_tok(const ChunkMeta &m, int src) {
    Tok k;
    k.pos = __shfl_sync(0xffffffffu, static_cast<long long>(m.pos), src);
    k.slot = __shfl_sync(0xffffffffu, static_cast<long long>(m.slot), src);
    k.req = __shfl_sync(0xffffffffu, m.req, src);
    k.q0 = __shfl_sync(0xffffffffu, m.q0, src);
    return k;
}

template <typename E, int VEC, int MAXW, int PF>
__global__ void __launch_bounds__(kThreads, MAXW <= 4 ? 2 : 1) fused_strip_kernel(const __grid_constant__ FusedArgs a) {
    using P = Pack<E, VEC>;
    constexpr int Q = Ring<PF, MAXW>::Q;
    static_assert(32 % Q == 0, "a metadata chunk holds whole ring turns");
    pdl_wait();
    pdl_trigger();
    const int nv = a.C / VEC;
    const int t_begin = (blockIdx.x * blockDim.y + threadIdx.y) * a.strip;
    if (t_begin >= a.T) return;  // uniform across the warp (one strip per warp row)
    // Lanes past the last channel pack stay in the loop (the metadata
    // shuffles need the full warp) but load a valid pack and store nothing.
    const int pack_raw = blockIdx.y * blockDim.x + threadIdx.x;
    const bool active = pack_raw < nv;
    const int pack = active ? pack_raw : nv - 1;
    const int lid = threadIdx.x & 31;
    const int t_end = t_begin + a.strip < a.T ? t_begin + a.strip : a.T;
    const E *x = static_cast<const E *>(a.x) + pack * VEC;  // column of this pack
    const int c = pack * VEC;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);

    P ring[Q];  // ring[(row - t_begin) mod Q] holds x row `row`
#pragma unroll
    for (int j = 0; j < PF; ++j)
        if (t_begin + j < t_end) ring[j].load_nc(x + static_cast<int64_t>(t_begin + j) * a.x_rs);
    ChunkMeta cur = load_chunk(a, t_begin + lid, t_end);
    float wr[MAXW][VEC];
    load_weights<E, VEC, MAXW>(a, c, wr);
    // Halo rows before the strip are same-forward taps only if the strip's
    // first token's request began earlier (a later token reaching back past
    // t_begin belongs to that same request).
    const int q0_first = __shfl_sync(0xffffffffu, cur.q0, 0);
#pragma unroll
    for (int d = 1; d < MAXW; ++d) {
        const int row = t_begin - d;
        if (d < a.W && row >= q0_first && row >= 0)
            ring[Q - d].load_nc(x + static_cast<int64_t>(row) * a.x_rs);
    }

    for (int cb = t_begin; cb < t_end; cb += 32) {
        const ChunkMeta nxt = load_chunk(a, cb + 32 + lid, t_end);
        const int c_end = cb + 32 < t_end ? cb + 32 : t_end;
        for (int base = cb; base < c_end; base += Q) {
#pragma unroll
            for (int j = 0; j < Q; ++j) {
                const int t = base + j;
                if (t >= c_end) break;
                const Tok k = shfl_tok(cur, t - cb);
                const int tn = t + PF;  // prefetch the x row PF tokens ahead
                if (tn < t_end) ring[(j + PF) % Q].load_nc(x + static_cast<int64_t>(tn) * a.x_rs);
                if (k.slot == -1) continue;  // PAD row

                unsigned bad = check_tok<false>(a, k, t);
                if (!bad && t - k.q0 >= a.W - 1) {
                    // Every tap is an x row of this step, already in the ring.
                    if (active)
                        conv_store<E, VEC, MAXW>(
                            a, wr,
                            [&](int d, bool &u) {
                                u = true;
                                return ring[(j - d + Q) % Q];
                            },
                            ring[j], t, c, k.slot, lane);
                    continue;
                }
                // The first W-1 tokens of a request: earlier taps from the
                // cache (or zero before position 0).
                P ct[MAXW];
                bool from_x[MAXW], use[MAXW];
#pragma unroll
                for (int d = 1; d < MAXW; ++d) {
                    from_x[d] = t - d >= k.q0;
                    use[d] = from_x[d] || k.pos - d >= 0;
                    if (d < a.W && !from_x[d] && k.pos - d >= 0 && !bad)
                        bad |= load_cache_tap<E, VEC>(a, k.req, k.pos - d, lane, ct[d]);
                }
                if (bad) {
                    if (a.err && active) atomicOr(a.err, static_cast<int>(bad));
                    continue;
                }
                if (active)
                    conv_store<E, VEC, MAXW>(
                        a, wr,
                        [&](int d, bool &u) {
                            u = d == 0 || use[d];
                            return (d == 0 || from_x[d]) ? ring[(j - d + Q) % Q] : ct[d];
                        },
                        ring[j], t, c, k.slot, lane);
            }
        }
        cur = nxt;
    }
}

struct Shape {
    int cv, tg;  // threads along channel packs, token rows (or strips) per block
};

inline int next_pow2(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

inline Shape block_shape(int nv, int64_t rows) {
    Shape s;
    s.cv = next_pow2(nv);
    if (s.cv < 32) s.cv = 32;
    if (s.cv > kThreads) s.cv = kThreads;
    int threads = kThreads;
    // Few rows: narrower blocks so more SMs get work.
    const int64_t blocks = ((rows + kThreads / s.cv - 1) / (kThreads / s.cv)) *
                           ((nv + s.cv - 1) / s.cv);
    if (blocks < 2 * 148 && s.cv <= 128) threads = 128;
    if (threads < s.cv) threads = s.cv;
    s.tg = threads / s.cv;
    return s;
}

// Speculative prefetching before the PDL wait pays off only when this
// launch's blocks can be resident while the preceding kernel still runs: a
// launch of at most an eighth of the GPU's thread slots (148 SMs x 2048).
// Measured (A/B, us, with / without): decode 256 x 128 threads 3.51 / 3.93,
// sconv_update 3.36 / 4.17; two streams in one launch (2 x 256 x 128
// threads) 4.56 / 4.47; spec decode 512 x 256 threads 7.57 / 6.12.
inline bool speculate(int64_t threads) { return threads <= 148LL * 256; }

// Strip kernel only when there is enough work to stream: T*C/VEC
// token-packs above this many.
constexpr int64_t kStripMinWork = 1 << 19;
constexpr int kPF = 4;

template <typename E, int VEC, int MAXW>
cudaError_t launch_w(FusedArgs &a, bool one, cudaStream_t stream) {
    // a.w_vec says the weight is a dense, 16-byte aligned [C, W].  The token
    // and strip kernels address it with the compile-time MAXW, so they take
    // vector loads only when W == MAXW; the tiled form uses the exact W and
    // takes them for every W.
    const int w_vec_exact = a.w_vec;
    a.w_vec = a.w_vec && a.W == MAXW;
    const int nv = a.C / VEC;
    const int64_t work = static_cast<int64_t>(a.T) * nv;
    if (one || work < kStripMinWork || a.T < 64) {
        const Shape s = block_shape(nv, a.T);
        dim3 grid(static_cast<unsigned>((a.T + s.tg - 1) / s.tg),
                  static_cast<unsigned>((nv + s.cv - 1) / s.cv));
        const bool spec =
            speculate(static_cast<int64_t>(grid.x) * grid.y * s.cv * s.tg);
        if (one)
            return spec ? launch_pdl(fused_token_kernel<E, VEC, MAXW, true, true>, grid,
                                     dim3(s.cv, s.tg), 0, stream, a)
                        : launch_pdl(fused_token_kernel<E, VEC, MAXW, true, false>, grid,
                                     dim3(s.cv, s.tg), 0, stream, a);
        return spec ? launch_pdl(fused_token_kernel<E, VEC, MAXW, false, true>, grid,
                                 dim3(s.cv, s.tg), 0, stream, a)
                    : launch_pdl(fused_token_kernel<E, VEC, MAXW, false, false>, grid,
                                 dim3(s.cv, s.tg), 0, stream, a);
    }
    if constexpr (VEC * sizeof(E) == 16) {
        FusedArgs tiled = a;
        tiled.w_vec = w_vec_exact;
        bool used = false;
        const cudaError_t e = launch_fused_tma(tiled, sizeof(E) == 2, stream, used);
        if (used || e != cudaSuccess) return e;
    }
    // Strip length: a whole number of 32-token metadata chunks, the longest
    // (up to 128 tokens) that still leaves about four waves of 256-thread
    // blocks on 148 SMs.
    int strip = 128;
    while (strip > 32 && (static_cast<int64_t>((a.T + strip - 1) / strip) * nv) < 4 * 148 * 2 * 256)
        strip /= 2;
    a.strip = strip;
    const int64_t strips = (a.T + strip - 1) / strip;
    const Shape s = block_shape(nv, strips);
    dim3 grid(static_cast<unsigned>((strips + s.tg - 1) / s.tg),
              static_cast<unsigned>((nv + s.cv - 1) / s.cv));
    return launch_pdl(fused_strip_kernel<E, VEC, MAXW, kPF>, grid, dim3(s.cv, s.tg), 0, stream, a);
}

template <typename E, int VEC>
cudaError_t launch_v(FusedArgs &a, bool one, cudaStream_t stream) {
    if (a.W <= 4) return launch_w<E, VEC, 4>(a, one, stream);
    return launch_w<E, VEC, 8>(a, one, stream);
}

template <typename E, int VEC, int MAXW>
cudaError_t launch_streams_t(FusedArgs *s, int n, cudaStream_t stream) {
    StreamSet m;
    m.n = n;
    int nv_max = 0;
    for (int i = 0; i < n; ++i) nv_max = s[i].C / VEC > nv_max ? s[i].C / VEC : nv_max;
    const Shape sh = block_shape(nv_max, s[0].T);
    m.y0[0] = 0;
    for (int i = 0; i < n; ++i) {
        s[i].w_vec = s[i].w_vec && s[i].W == MAXW;
        m.s[i] = s[i];
        m.y0[i + 1] = m.y0[i] + (s[i].C / VEC + sh.cv - 1) / sh.cv;
    }
    for (int i = n; i < SCONV_MAX_STREAMS; ++i) m.s[i] = s[0];  // never selected
    dim3 grid(static_cast<unsigned>((s[0].T + sh.tg - 1) / sh.tg), static_cast<unsigned>(m.y0[n]));
    if (speculate(static_cast<int64_t>(grid.x) * grid.y * sh.cv * sh.tg))
        return launch_pdl(fused_streams_kernel<E, VEC, MAXW, true>, grid, dim3(sh.cv, sh.tg), 0,
                          stream, m);
    return launch_pdl(fused_streams_kernel<E, VEC, MAXW, false>, grid, dim3(sh.cv, sh.tg), 0,
                      stream, m);
}

template <typename E, int VEC>
cudaError_t launch_streams_v(FusedArgs *s, int n, cudaStream_t stream) {
    if (s[0].W <= 4) return launch_streams_t<E, VEC, 4>(s, n, stream);
    return launch_streams_t<E, VEC, 8>(s, n, stream);
}

template <typename E, int VEC, int MAXW>
cudaError_t launch_taps_t(FusedArgs *s, int n, bool ready, cudaStream_t stream) {
    StreamSet m;
    m.n = n;
    int nv_max = 0;
    for (int i = 0; i < n; ++i) nv_max = s[i].C / VEC > nv_max ? s[i].C / VEC : nv_max;
    const Shape sh = block_shape(nv_max, s[0].T);
    m.y0[0] = 0;
    for (int i = 0; i < n; ++i) {
        s[i].w_vec = s[i].w_vec && s[i].W == MAXW;
        m.s[i] = s[i];
        m.y0[i + 1] = m.y0[i] + (s[i].C / VEC + sh.cv - 1) / sh.cv;
    }
    for (int i = n; i < SCONV_MAX_STREAMS; ++i) m.s[i] = s[0];  // never selected
    dim3 grid(static_cast<unsigned>((s[0].T + sh.tg - 1) / sh.tg), static_cast<unsigned>(m.y0[n]));
    const dim3 block(sh.cv, sh.tg);
    if (n == 1)
        return ready ? launch_pdl(fused_taps_kernel<E, VEC, MAXW, true>, grid, block, 0, stream,
                                  m.s[0])
                     : launch_pdl(fused_taps_kernel<E, VEC, MAXW, false>, grid, block, 0, stream,
                                  m.s[0]);
    return ready ? launch_pdl(fused_taps_streams_kernel<E, VEC, MAXW, true>, grid, block, 0,
                              stream, m)
                 : launch_pdl(fused_taps_streams_kernel<E, VEC, MAXW, false>, grid, block, 0,
                              stream, m);
}

template <typename E, int VEC, int MAXW>
cudaError_t launch_taps_next_t(FusedArgs *s, int n, TapResolveArgs &nx, cudaStream_t stream) {
    StreamSet m;
    m.n = n;
    int nv_max = 0;
    for (int i = 0; i < n; ++i) nv_max = s[i].C / VEC > nv_max ? s[i].C / VEC : nv_max;
    // Large blocks even for few rows: measured on the decode step (256
    // tokens x 128 packs, us per launch), 256 blocks of 128 threads 2.90,
    // 128 of 256 2.79, 64 of 512 (one stream) 2.785 against 2.827 in
    // another session.  Several streams keep kThreads.
    Shape sh = block_shape(nv_max, s[0].T);
    const int want = n == 1 ? kNextThreads : kThreads;
    if (sh.cv * sh.tg < want) sh.tg = want / sh.cv;
    m.y0[0] = 0;
    for (int i = 0; i < n; ++i) {
        s[i].w_vec = s[i].w_vec && s[i].W == MAXW;
        m.s[i] = s[i];
        m.y0[i + 1] = m.y0[i] + (s[i].C / VEC + sh.cv - 1) / sh.cv;
    }
    for (int i = n; i < SCONV_MAX_STREAMS; ++i) m.s[i] = s[0];  // never selected
    const int gx = (s[0].T + sh.tg - 1) / sh.tg;
    const int threads = sh.cv * sh.tg;
    const int bx = (nx.num_padded + threads - 1) / threads;  // build blocks
    size_t smem = 0;
    resolve_staging(nx, smem);
    const dim3 grid(static_cast<unsigned>(gx + bx), static_cast<unsigned>(m.y0[n]));
    const dim3 block(sh.cv, sh.tg);
    const bool dec = nx.qsl == nullptr;
    if (n == 1)
        return dec ? launch_pdl(fused_taps_next_kernel<E, VEC, MAXW, true>, grid, block, smem,
                                stream, m.s[0], nx, gx)
                   : launch_pdl(fused_taps_next_kernel<E, VEC, MAXW, false>, grid, block, smem,
                                stream, m.s[0], nx, gx);
    return dec ? launch_pdl(fused_taps_streams_next_kernel<E, VEC, MAXW, true>, grid, block, smem,
                            stream, m, nx, gx)
               : launch_pdl(fused_taps_streams_next_kernel<E, VEC, MAXW, false>, grid, block,
                            smem, stream, m, nx, gx);
}

template <typename E, int VEC>
cudaError_t launch_taps_next_v(FusedArgs *s, int n, TapResolveArgs &nx, cudaStream_t stream) {
    if (s[0].W <= 4) return launch_taps_next_t<E, VEC, 4>(s, n, nx, stream);
    return launch_taps_next_t<E, VEC, 8>(s, n, nx, stream);
}

template <typename E, int VEC>
cudaError_t launch_taps_v(FusedArgs *s, int n, bool ready, cudaStream_t stream) {
    if (s[0].W <= 4) return launch_taps_t<E, VEC, 4>(s, n, ready, stream);
    return launch_taps_t<E, VEC, 8>(s, n, ready, stream);
}

}  // namespace

cudaError_t launch_fused_streams(FusedArgs *s, int n, bool bf16_data, bool vec,
                                 cudaStream_t stream) {
    // Prefill sizes are bandwidth-bound and nothing is gained by sharing
    // the metadata: each stream takes its own (streamed or TMA) launch.
    int64_t packs = 0;
    for (int i = 0; i < n; ++i) packs += s[i].C / (vec ? (bf16_data ? 8 : 4) : 1);
    if (static_cast<int64_t>(s[0].T) * packs >= kStripMinWork && s[0].T >= 64) {
        for (int i = 0; i < n; ++i) {
            const cudaError_t e = launch_fused(s[i], bf16_data, vec, false, stream);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    for (int i = 0; i < n; ++i) {
        s[i].divN = FastDiv::make(static_cast<uint32_t>(s[i].N));
        s[i].slots32 = s[i].num_blocks * s[i].N < (1ll << 31);
        s[i].strip = 1;
    }
    if (bf16_data)
        return vec ? launch_streams_v<bf16, 8>(s, n, stream) : launch_streams_v<bf16, 1>(s, n, stream);
    return vec ? launch_streams_v<float, 4>(s, n, stream) : launch_streams_v<float, 1>(s, n, stream);
}

cudaError_t launch_fused_taps(FusedArgs *s, int n, bool bf16_data, bool vec, bool ready,
                              cudaStream_t stream) {
    for (int i = 0; i < n; ++i) {
        s[i].divN = FastDiv::make(static_cast<uint32_t>(s[i].N));
        s[i].slots32 = s[i].num_blocks * s[i].N < (1ll << 31);
        s[i].strip = 1;
    }
    // Prefill sizes of one stream: the TMA-pipelined kernel, which reads the
    // tile's table rows with its x rows (the same bits as the token form).
    const int vec_n = bf16_data ? 8 : 4;
    if (n == 1 && vec && s[0].T >= 64 &&
        static_cast<int64_t>(s[0].T) * (s[0].C / vec_n) >= kStripMinWork) {
        bool used = false;
        const cudaError_t e = launch_fused_tma_taps(s[0], bf16_data, stream, used);
        if (used || e != cudaSuccess) return e;
    }
    if (bf16_data)
        return vec ? launch_taps_v<bf16, 8>(s, n, ready, stream)
                   : launch_taps_v<bf16, 1>(s, n, ready, stream);
    return vec ? launch_taps_v<float, 4>(s, n, ready, stream)
               : launch_taps_v<float, 1>(s, n, ready, stream);
}

cudaError_t launch_fused_taps_next(FusedArgs *s, int n, bool bf16_data, bool vec,
                                   TapResolveArgs &next, cudaStream_t stream) {
    for (int i = 0; i < n; ++i) {
        s[i].divN = FastDiv::make(static_cast<uint32_t>(s[i].N));
        s[i].slots32 = s[i].num_blocks * s[i].N < (1ll << 31);
        s[i].strip = 1;
    }
    if (bf16_data)
        return vec ? launch_taps_next_v<bf16, 8>(s, n, next, stream)
                   : launch_taps_next_v<bf16, 1>(s, n, next, stream);
    return vec ? launch_taps_next_v<float, 4>(s, n, next, stream)
               : launch_taps_next_v<float, 1>(s, n, next, stream);
}

cudaError_t launch_fused(FusedArgs &a, bool bf16_data, bool vec, bool one, cudaStream_t stream) {
    a.divN = FastDiv::make(static_cast<uint32_t>(a.N));
    a.slots32 = a.num_blocks * a.N < (1ll << 31);
    a.strip = 1;
    if (bf16_data) {
        return vec ? launch_v<bf16, 8>(a, one, stream) : launch_v<bf16, 1>(a, one, stream);
    }
    return vec ? launch_v<float, 4>(a, one, stream) : launch_v<float, 1>(a, one, stream);
}

}  // namespace sconv
