// dense.cu -- the dense-state interface of the short convolution, sm_100a
// ("Implementation:Sgl project Sglang Mamba Ops": causal_conv1d_fwd and
// causal_conv1d_update).  A sequence's history is a dense line of its last L
// inputs (oldest first) instead of the paged cache, and x, out and the lines
// may all be updated in place.
//
//  * dense_fwd_tile -- varlen prefill, x token-major in 16-byte channel
//    packs.  One 256-thread block owns a (sequence, column of PP packs) and
//    walks it in tiles of TT = 2 * 256 / PP rows, which one thread brings
//    into a shared-memory ring by tensor copy four or five tiles ahead;
//    per-stage mbarriers pace the copies and the eight warps, with no
//    block-wide barrier per tile.  Each thread convolves two rows of the
//    current tile.  Each ring stage holds the W-1 rows before its tile,
//    written while the previous tile is computed; the new state line is
//    read from the last two tiles at the end.  No block re-reads x rows
//    that another block may already have overwritten, so the in-place form
//    needs no scratch memory and no ordering between blocks.  PP is chosen
//    per call: the widest column that still gives the SMs 1.5 blocks each,
//    and blocks run longest sequence first.
//  * dense_fwd_cm -- channel-major x (token stride 1): a warp per (sequence,
//    channel) walks the channel's contiguous tokens, one 16-byte vector (8
//    bf16 or 4 fp32 tokens) per lane, with the taps before a lane's tokens
//    shuffled from the lanes below.
//  * dense_fwd_generic -- any other layout: a thread per (sequence, channel)
//    walks the rows with the taps in registers.
//  * dense_update -- one token per sequence; shifted or circular line.
//
// Every sum runs oldest tap first, starting from the bias, in fp32 FMAs, so
// all the kernels agree bit for bit on the same token.  A sequence whose
// line or row range is out of range is skipped and reported through the
// optional error flag; nothing traps, and the tiled prefill's mbarrier
// waits are bounded in time (SCONV_EFLAG_TIMEOUT).
#include <mutex>

#include "common.cuh"
#include "sconv.h"
#include "tma.cuh"

namespace sconv {
namespace {

constexpr int kRowsPerThread = 2;  // rows of a tile each thread convolves
constexpr int kTileThreads = 256;
// Ring depth of the tiled prefill: 5 stages when the grid runs in several
// waves of blocks (many sequences: short columns, where a deep ring only
// fetches ahead of the end), 6 when the blocks fit in about one wave (long
// columns that must stream at full rate).  Measured on the dense mixed and
// long prefills (us): 4 / 6 stages 49.7 / 404, 5 / 5: 49.3 / 425, 6 / 8:
// 49.4 / 405.
constexpr int kStagesFew = 5;
constexpr int kStagesMany = 6;
constexpr int kLptMaxBatch = 64;   // longest-first block order up to this many sequences
constexpr int kMaxL = SCONV_MAX_STATE_LEN;

template <typename E>
struct RawOf;
template <>
struct RawOf<bf16> {
    using T = uint16_t;
};
template <>
struct RawOf<float> {
    using T = uint32_t;
};

// VEC raw elements moved as one load or store of VEC * sizeof(R) bytes.
template <int BYTES>
struct RawVec;
template <>
struct RawVec<2> {
    using T = uint16_t;
};
template <>
struct RawVec<4> {
    using T = uint32_t;
};
template <>
struct RawVec<8> {
    using T = uint2;
};
template <>
struct RawVec<16> {
    using T = uint4;
};
template <typename R, int VEC>
union Lanes {
    typename RawVec<VEC * sizeof(R)>::T v;
    R e[VEC];
};

__device__ __forceinline__ float raw_to_float(uint16_t v) {
    return __uint_as_float(static_cast<uint32_t>(v) << 16);
}
__device__ __forceinline__ float raw_to_float(uint32_t v) { return __uint_as_float(v); }

template <typename E>
__device__ __forceinline__ typename RawOf<E>::T float_to_raw(float f);
template <>
__device__ __forceinline__ uint16_t float_to_raw<bf16>(float f) {
    const bf16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<const uint16_t *>(&h);
}
template <>
__device__ __forceinline__ uint32_t float_to_raw<float>(float f) {
    return __float_as_uint(f);
}

__device__ __forceinline__ void flag(int32_t *err, unsigned bits) {
    if (err) atomicOr(err, static_cast<int>(bits));
}

// Per-sequence checks shared by the prefill kernels.  Returns false (after
// flagging, from one thread of the sequence) when the sequence is skipped;
// otherwise sets the row range, the line and whether the history comes from
// the line.
__device__ __forceinline__ bool sequence_setup(const DenseArgs &a, int b, bool reporter,
                                               int &q0, int &n, int64_t &line, bool &from) {
    q0 = __ldg(a.qsl + b);
    const int q1 = __ldg(a.qsl + b + 1);
    if (q0 < 0 || q1 < q0 || q1 > a.T) {
        if (reporter) flag(a.err, SCONV_EFLAG_QUERY_START);
        return false;
    }
    n = q1 - q0;
    line = a.lines ? __ldg(a.lines + b) : b;
    if (a.lines && line == a.pad) return false;  // padded entry
    if (a.st && (line < 0 || line >= a.num_lines)) {
        if (reporter) flag(a.err, SCONV_EFLAG_SLOT);
        return false;
    }
    from = a.st && a.init && __ldg(a.init + b);
    return true;
}

// Weights of VEC channels from c, indexed by tap slot k' in 0..MAXW-1 with
// tap k = k' - (MAXW - W); slots before the first tap hold zero.
template <typename E, int VEC, int MAXW>
__device__ __forceinline__ void load_taps(const DenseArgs &a, int c, float (&w)[MAXW][VEC]) {
    const E *wp = static_cast<const E *>(a.w);
#pragma unroll
    for (int kk = 0; kk < MAXW; ++kk) {
        const int k = kk - (MAXW - a.W);
#pragma unroll
        for (int v = 0; v < VEC; ++v)
            w[kk][v] = k >= 0 ? load_weight(wp + (c + v) * a.w_sc + k * a.w_sk) : 0.f;
    }
}

template <typename E, int VEC>
__device__ __forceinline__ void load_bias(const DenseArgs &a, int c, float (&acc)[VEC]) {
    const E *bp = static_cast<const E *>(a.bias);
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = bp ? load_weight(bp + c + v) : 0.f;
}

// State line entry i of VEC channels from c, as one raw pack (zero when the
// history does not come from the line).
template <typename E, int VEC>
__device__ __forceinline__ uint4 line_pack(const DenseArgs &a, int64_t line, int c, int i,
                                           bool from) {
    using R = typename RawOf<E>::T;
    union {
        uint4 u;
        R e[VEC];
    } p;
    p.u = make_uint4(0u, 0u, 0u, 0u);
    if (from) {
        const R *s = static_cast<const R *>(a.st) + line * a.s_line + i * a.s_k;
#pragma unroll
        for (int v = 0; v < VEC; ++v) p.e[v] = s[static_cast<int64_t>(c + v) * a.s_c];
    }
    return p.u;
}

template <typename E, int VEC>
__device__ __forceinline__ void store_line_pack(const DenseArgs &a, int64_t line, int c, int i,
                                                uint4 u) {
    using R = typename RawOf<E>::T;
    union {
        uint4 u;
        R e[VEC];
    } p;
    p.u = u;
    R *s = static_cast<R *>(a.st) + line * a.s_line + i * a.s_k;
#pragma unroll
    for (int v = 0; v < VEC; ++v) s[static_cast<int64_t>(c + v) * a.s_c] = p.e[v];
}

// acc[v] += w[v] * tap[v] for the eight bf16 channels of a pack, with the
// mixed-precision FMA that takes bf16 operands directly: the product of two
// bf16 values is exact in fp32, so this equals widening both and one fmaf,
// bit for bit.  w holds the weights of one tap as four bf16 pairs (channel
// 2i in the low half), the same layout as the pack's words.
__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], const uint32_t (&w)[4], uint4 tap) {
    const uint32_t q[4] = {tap.x, tap.y, tap.z, tap.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{\n\t.reg .b16 wl, wh, tl, th;\n\t"
            "mov.b32 {wl, wh}, %2;\n\t"
            "mov.b32 {tl, th}, %3;\n\t"
            "fma.rn.f32.bf16 %0, wl, tl, %0;\n\t"
            "fma.rn.f32.bf16 %1, wh, th, %1;\n\t}"
            : "+f"(acc[2 * i]), "+f"(acc[2 * i + 1])
            : "r"(w[i]), "r"(q[i]));
}

// Per-thread weights of the tiled kernel: bf16 pairs for bf16 data, floats
// for fp32 data; tap slot k' as in load_taps.
template <typename E, int MAXW>
struct TileWeights {
    float w[MAXW][4];
    __device__ __forceinline__ void load(const DenseArgs &a, int c) {
        load_taps<float, 4, MAXW>(a, c, w);
    }
    __device__ __forceinline__ void fma(float (&acc)[4], int kk, uint4 tap) const {
        const float t[4] = {__uint_as_float(tap.x), __uint_as_float(tap.y),
                            __uint_as_float(tap.z), __uint_as_float(tap.w)};
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[v] = fmaf(w[kk][v], t[v], acc[v]);
    }
};
template <int MAXW>
struct TileWeights<bf16, MAXW> {
    uint32_t w[MAXW][4];
    __device__ __forceinline__ void load(const DenseArgs &a, int c) {
        const uint16_t *wp = static_cast<const uint16_t *>(a.w);
#pragma unroll
        for (int kk = 0; kk < MAXW; ++kk) {
            const int k = kk - (MAXW - a.W);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t lo = 0, hi = 0;
                if (k >= 0) {
                    lo = __ldg(wp + (c + 2 * i) * a.w_sc + k * a.w_sk);
                    hi = __ldg(wp + (c + 2 * i + 1) * a.w_sc + k * a.w_sk);
                }
                w[kk][i] = lo | (hi << 16);
            }
        }
    }
    __device__ __forceinline__ void fma(float (&acc)[8], int kk, uint4 tap) const {
        fma_bf16x8(acc, w[kk], tap);
    }
};

// Two independent fp32 products (d_i = a_i * b_i, each rounded once) in one
// packed sm_100 instruction.
__device__ __forceinline__ void mul2(float &d0, float &d1, float a0, float a1, float b0,
                                     float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// The activation of VEC accumulators in place.  bf16 data: the operations
// of silu<bf16> (h = y/2, then h + h*tanh(h)) with the multiply and the FMA
// done two at a time in packed fp32 instructions -- the same roundings, so
// the same bits as the scalar form the other kernels use.
template <typename E, int VEC>
__device__ __forceinline__ void silu_pack(float (&acc)[VEC]) {
    if constexpr (sizeof(E) == 2) {
        float h[VEC], t[VEC];
#pragma unroll
        for (int v = 0; v < VEC; v += 2) mul2(h[v], h[v + 1], acc[v], acc[v + 1], 0.5f, 0.5f);
#pragma unroll
        for (int v = 0; v < VEC; ++v) asm("tanh.approx.f32 %0, %1;" : "=f"(t[v]) : "f"(h[v]));
#pragma unroll
        for (int v = 0; v < VEC; v += 2) {
            acc[v] = h[v];
            acc[v + 1] = h[v + 1];
            fma2(acc[v], acc[v + 1], h[v], h[v + 1], t[v], t[v + 1]);
        }
    } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = silu<E>(acc[v]);
    }
}

// Prefill, token-major x.  Block i covers column y of sequence b (packs
// y*PP .. y*PP+PP-1); with at most kLptMaxBatch sequences the blocks go
// longest sequence first (so the long columns start in the first wave and
// short ones fill the tail), else sequences interleave.  A tile is TT rows;
// thread (g, p) = (threadIdx.x / PP, threadIdx.x % PP) convolves rows
// g*RPT .. g*RPT+RPT-1 of pack p from a register window of W-1+RPT rows.
//
// Tiles arrive by tensor copy: thread 0 issues each tile's TT x PP-pack box
// into a ring stage and the copy completes on the stage's `full` mbarrier;
// each warp releases the stage on its `empty` mbarrier when it is done, and
// thread 0 refills the stage of tile s-1 (once all eight warps released it)
// after tile s, so a warp never waits for the others to finish the tile it
// is on and no block-wide barrier runs per tile.  Each stage keeps the WT-1
// rows before its tile (the halo) just below the tile's rows: only warp 0
// reads them (the first rows of a tile), and warp 0 writes them, from the
// last rows of the previous tile (the first from the state line), so every
// tap is a plain shared-memory read and the halo needs only warp-level
// ordering.  The new state line, the last L inputs, is read at the end from
// the last two tiles' stages (TT >= L) and the old line kept in shared
// memory.  Copies cover whole tiles and may read rows past the sequence's
// end (another sequence's, possibly being rewritten in place by its own
// block, or zeros past T); those rows are never used.  Rows of this
// sequence are copied before this block writes them, and never re-read, so
// the in-place form needs no scratch memory and no ordering between blocks.
// WT is the exact tap count (2..4), or 8 for any W up to 8.
template <int PP, int WT, int THREADS, int STAGES>
struct TileLayout {
    static constexpr int TT = THREADS / PP * kRowsPerThread;
    static constexpr int HALO = WT - 1;
    static constexpr int row_bytes = PP * 16;
    // The tile's rows start on a 128-byte boundary (the copy's destination);
    // the halo rows sit just below them.
    static constexpr int tile_off = (HALO * row_bytes + 127) / 128 * 128;
    static constexpr int halo_off = tile_off - HALO * row_bytes;
    static constexpr int stage = tile_off + TT * row_bytes;
    static constexpr int tile_bytes = TT * row_bytes;
    // A copy box holds at most 256 rows.
    static constexpr int boxes = TT > 256 ? TT / 256 : 1;
    static constexpr int box_rows = TT / boxes;
    static constexpr int bars = STAGES * stage;  // full[STAGES], empty[STAGES]
    static constexpr int line0 = bars + 2 * STAGES * 8;
    static constexpr int order = line0 + kMaxL * PP * 16;
    static constexpr int smem = order + kLptMaxBatch * 4;
};

template <typename E, int PP, int WT, int THREADS, int STAGES>
__global__ void __launch_bounds__(THREADS)
dense_fwd_tile(const __grid_constant__ DenseArgs a, const __grid_constant__ CUtensorMap xmap,
               int ncb) {
    using Lay = TileLayout<PP, WT, THREADS, STAGES>;
    using namespace tma;
    constexpr int VEC = 16 / sizeof(E);
    constexpr int RPT = kRowsPerThread;
    constexpr int TT = Lay::TT;
    constexpr int HALO = Lay::HALO;
    constexpr int NW = WT - 1 + RPT;  // window rows of one thread
    // The threads whose windows reach into the halo are all in warp 0.
    static_assert((HALO + RPT - 1) / RPT * PP <= 32, "halo readers must be warp 0");
    static_assert(TT >= kMaxL, "the new line must lie in the last two tiles");
    static_assert(STAGES >= 3, "the halo stage must differ from the refilled one");
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Lay::bars);
    uint64_t *empty = full + STAGES;
    uint4 *line0 = reinterpret_cast<uint4 *>(smem + Lay::line0);  // the old line, L x PP
    int *order = reinterpret_cast<int *>(smem + Lay::order);
    // Row -HALO of stage k: the halo, then the tile's TT rows, PP packs each.
    auto rows = [&](int k) { return reinterpret_cast<uint4 *>(smem + k * Lay::stage + Lay::halo_off); };

    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int k = 0; k < STAGES; ++k) {
            mbar_init(&full[k], 1);
            mbar_init(&empty[k], THREADS / 32);
        }
        mbar_init_fence();
    }
    int b, y;
    if (a.batch <= kLptMaxBatch) {
        // Rank sequences by length, longest first (ties by index).
        if (threadIdx.x < a.batch) {
            const int t = threadIdx.x;
            const int len = __ldg(a.qsl + t + 1) - __ldg(a.qsl + t);
            int rank = 0;
            for (int u = 0; u < a.batch; ++u) {
                const int lu = __ldg(a.qsl + u + 1) - __ldg(a.qsl + u);
                rank += (lu > len) || (lu == len && u < t);
            }
            order[rank] = t;
        }
        __syncthreads();  // the ranking and the barriers
        b = order[blockIdx.x / ncb];
        y = blockIdx.x % ncb;
    } else {
        __syncthreads();  // the barriers
        b = blockIdx.x % a.batch;
        y = blockIdx.x / a.batch;
    }
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int p = threadIdx.x % PP;
    const int g = threadIdx.x / PP;
    const int c = (y * PP + p) * VEC;
    const bool cvalid = c < a.dim;
    const int W = WT == 8 ? a.W : WT;

    int q0, n;
    int64_t line;
    bool from;
    if (!sequence_setup(a, b, threadIdx.x == 0 && y == 0, q0, n, line, from)) return;
    const int L = a.L;
    const int ntiles = (n + TT - 1) / TT;
    const int cx = y * PP * VEC;  // the column's first channel

    // Thread 0 is the producer: it puts tile j in stage j % STAGES.
    int issued = 0;  // tiles issued (thread 0)
    auto issue = [&](int j) {
        const int k = j % STAGES;
        unsigned char *dst = smem + k * Lay::stage + Lay::tile_off;
        mbar_expect_tx(&full[k], Lay::tile_bytes);
#pragma unroll
        for (int bx = 0; bx < Lay::boxes; ++bx)
            copy_2d(dst + bx * Lay::box_rows * Lay::row_bytes, &xmap, cx,
                    q0 + j * TT + bx * Lay::box_rows, &full[k]);
        issued = j + 1;
    };
    if (threadIdx.x == 0)
        for (int j = 0; j < STAGES && j < ntiles; ++j) issue(j);

    // The history: the old line (or zeros), and its last HALO entries as the
    // first tile's halo (zeros before the line).
    const int ci = threadIdx.x / PP;  // line entry / halo row this thread sets up
    if (a.st && ci < L)
        line0[ci * PP + p] = cvalid ? line_pack<E, VEC>(a, line, c, ci, from)
                                    : make_uint4(0u, 0u, 0u, 0u);
    if (ci < HALO) {
        const int e = L - HALO + ci;
        rows(0)[ci * PP + p] = (cvalid && a.st && e >= 0) ? line_pack<E, VEC>(a, line, c, e, from)
                                                          : make_uint4(0u, 0u, 0u, 0u);
    }

    TileWeights<E, WT> wt;
    float bias[VEC];
    if (cvalid) {
        wt.load(a, c);
        load_bias<E, VEC>(a, c, bias);
    }
    __syncthreads();  // the old line and the first halo

    E *out = static_cast<E *>(a.out) + static_cast<int64_t>(q0) * a.x_st + c;
    const int r0 = g * RPT;
    bool alive = true;
    int next = 0;  // tiles this thread has waited for
    for (int s = 0; s < ntiles; ++s) {
        const int k = s % STAGES;
        const bool ok = mbar_wait(&full[k], (s / STAGES) & 1);
        if (!__all_sync(0xffffffffu, ok)) {  // the copy did not arrive in time
            if (lane == 0) flag(a.err, SCONV_EFLAG_TIMEOUT);
            alive = false;
            break;
        }
        next = s + 1;
        const uint4 *stage = rows(k);  // row -HALO of the tile
        // Warp 0: the next tile's halo, the last HALO rows of this (full) tile.
        if (warp == 0 && s + 1 < ntiles) {
            uint4 *h = rows((s + 1) % STAGES);
            for (int i = lane; i < HALO * PP; i += 32) h[i] = stage[TT * PP + i];
        }
        const int nv = min(TT, n - s * TT);
        if (r0 < nv && cvalid) {
            // win[j] holds tile row r0 - (WT-1) + j.
            uint4 win[NW];
#pragma unroll
            for (int j = 0; j < NW; ++j) {
                if (j < WT - W) continue;  // before the first tap of row r0
                win[j] = stage[(r0 + j) * PP + p];
            }
            E *orow = out + static_cast<int64_t>(s * TT + r0) * a.x_st;
#pragma unroll
            for (int u = 0; u < RPT; ++u) {
                if (r0 + u >= nv) break;
                float acc[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = bias[v];
#pragma unroll
                for (int kk = 0; kk < WT; ++kk)
                    if (kk >= WT - W) wt.fma(acc, kk, win[u + kk]);
                if (a.silu) silu_pack<E, VEC>(acc);
                Pack<E, VEC> o;
                o.from_float(acc);
                o.store(orow + u * a.x_st);
            }
        }
        // This warp is done with the stage (and warp 0's halo writes are
        // ordered before its next tile's reads).
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[k]);
        // Warp 0: refill the stage of tile s-1 once every warp released it.
        if (warp == 0) {
            bool fine = true;
            if (lane == 0 && s >= 1 && s - 1 + STAGES < ntiles) {
                const int j = s - 1;
                fine = mbar_wait(&empty[j % STAGES], (j / STAGES) & 1);
                if (fine) issue(j + STAGES);
            }
            if (!__shfl_sync(0xffffffffu, fine, 0)) {
                if (lane == 0) flag(a.err, SCONV_EFLAG_TIMEOUT);
                alive = false;
                break;
            }
        }
    }
    if (!alive) {
        // Let the copies issued and not waited for land before the block's
        // shared memory is released (each wait bounded); store nothing more.
        if (threadIdx.x == 0)
            for (int j = next; j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
        return;
    }
    // The new line: entry ci is input n + ci of (old line, the n rows).
    if (a.st && ci < L && cvalid) {
        const int i = n + ci;
        uint4 v;
        if (i < L) {
            v = line0[i * PP + p];
        } else {
            const int r = i - L;  // a row of the last two tiles
            v = rows((r / TT) % STAGES)[(HALO + r % TT) * PP + p];
        }
        store_line_pack<E, VEC>(a, line, c, ci, v);
    }
}

// Prefill, channel-major x (token stride 1).  Warp (b, c) walks channel c of
// sequence b in chunks of 32 * TOK tokens, lane l holding TOK consecutive
// tokens (one 16-byte vector) of a chunk.  The chunks are aligned to 16-byte
// boundaries of the row, so a sequence that starts mid-vector has its first
// `skew` slots masked: those read the state line (or zero) instead of x, and
// are not written.  The W-1 tokens before a lane's first come from the lanes
// below it (for the lowest lanes, from the previous chunk, or from the state
// line for the first) by shuffles.  Chunks are loaded kCmAhead ahead.  A warp
// reads a chunk before it writes it and never reads a chunk it has written,
// so the in-place form is safe; masked slots may belong to a neighbouring
// sequence, whose warp may be writing them, and are never used.  The sums
// run oldest tap first from the bias, as in the other kernels.
constexpr int kCmAhead = 4;  // chunks loaded ahead

template <typename E, int MAXW>
__global__ void __launch_bounds__(256) dense_fwd_cm(const __grid_constant__ DenseArgs a) {
    using R = typename RawOf<E>::T;
    constexpr int TOK = 16 / sizeof(R);  // tokens per lane
    constexpr int CHUNK = 32 * TOK;      // tokens per warp chunk
    constexpr unsigned kFull = 0xffffffffu;
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const bool live = gw < static_cast<int64_t>(a.batch) * a.dim;
    const int b = static_cast<int>(gw / a.dim);
    const int c = static_cast<int>(gw - static_cast<int64_t>(b) * a.dim);
    const int W = a.W, L = a.L;
    // The weights are constant: loaded while the preceding kernel drains.
    // wl[d] multiplies the token d back (weight column W-1-d).
    float wl[MAXW];
    float bias = 0.f;
    if (live) {
        const E *wp = static_cast<const E *>(a.w) + static_cast<int64_t>(c) * a.w_sc;
#pragma unroll
        for (int d = 0; d < MAXW; ++d) wl[d] = d < W ? load_weight(wp + (W - 1 - d) * a.w_sk) : 0.f;
        if (a.bias) bias = load_weight(static_cast<const E *>(a.bias) + c);
    }
    pdl_wait();
    pdl_trigger();
    if (!live) return;
    int q0, n;
    int64_t line;
    bool from;
    if (!sequence_setup(a, b, lane == 0 && c == 0, q0, n, line, from)) return;

    R *st = a.st ? static_cast<R *>(a.st) + line * a.s_line + static_cast<int64_t>(c) * a.s_c
                 : nullptr;
    // Token t of the sequence (t < 0: the history) as it enters the taps.
    auto history = [&](int t) -> float {
        const int h = L + t;  // line entry
        return (from && h >= 0) ? raw_to_float(st[static_cast<int64_t>(h) * a.s_k]) : 0.f;
    };

    const int64_t base = static_cast<int64_t>(c) * a.x_sc + static_cast<int64_t>(q0) * a.x_st;
    const R *xrow = static_cast<const R *>(a.x) + base;
    R *orow = static_cast<R *>(a.out) + base;
    // Slots of the first vector before the sequence's first token (x itself
    // is 16-byte aligned: the host sends other layouts elsewhere).
    const int skew = static_cast<int>((reinterpret_cast<uintptr_t>(xrow) / sizeof(R)) % TOK);
    const bool aligned_out = ((reinterpret_cast<uintptr_t>(orow) / sizeof(R)) % TOK) == skew &&
                             (reinterpret_cast<uintptr_t>(orow) % sizeof(R)) == 0;
    const int nchunks = (n + skew + CHUNK - 1) / CHUNK;
    const R *xv = xrow - skew;  // 16-byte aligned
    R *ov = orow - skew;

    // This lane's vector of chunk k.  A whole 16-byte load only when the
    // vector ends inside the sequence (its start may lie before it: those
    // slots are still inside x, since x is 16-byte aligned, and are replaced
    // by the history); otherwise single elements of the sequence only, so
    // nothing past the sequence's last token is read.
    auto fetch = [&](int k) -> uint4 {
        const int t0 = k * CHUNK - skew + TOK * lane;
        if (t0 + TOK <= n) return *reinterpret_cast<const uint4 *>(xv + k * CHUNK + TOK * lane);
        Lanes<R, TOK> v;
        v.v = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < TOK; ++i)
            if (t0 + i >= 0 && t0 + i < n) v.e[i] = xrow[t0 + i];
        return v.v;
    };
    // x first: its loads do not wait for the line's.
    uint4 buf[kCmAhead];
#pragma unroll
    for (int u = 0; u < kCmAhead; ++u)
        if (u < nchunks) buf[u] = fetch(u);
    // Every read of the old line comes before any write to it.  prv: this
    // lane's slots of the previous chunk (before the first chunk, the
    // history); head: the first chunk's slots before the sequence (the
    // history); keep: the entries that survive the call (n < L: new entry i
    // = old entry n + i).
    float prv[TOK], head[TOK];
#pragma unroll
    for (int i = 0; i < TOK; ++i) {
        prv[i] = history(TOK * lane + i - CHUNK - skew);
        const int t = TOK * lane + i - skew;
        head[i] = t < 0 ? history(t) : 0.f;
    }
    if (st) {
        const bool mine = lane < L && n + lane < L;
        R keep = R(0);
        if (mine && from) keep = st[static_cast<int64_t>(n + lane) * a.s_k];
        __syncwarp();  // the old line is read (by every lane) before any entry is written
        if (mine) st[static_cast<int64_t>(lane) * a.s_k] = keep;
    }

    for (int k0 = 0; k0 < nchunks; k0 += kCmAhead) {
#pragma unroll
        for (int u = 0; u < kCmAhead; ++u) {
            const int k = k0 + u;
            if (k >= nchunks) break;
            Lanes<R, TOK> cur;
            cur.v = buf[u];
            if (k + kCmAhead < nchunks) buf[u] = fetch(k + kCmAhead);  // never a chunk it wrote
            const int t0 = k * CHUNK - skew + TOK * lane;  // sequence index of slot 0
            const bool full = k * CHUNK >= skew && (k + 1) * CHUNK - skew <= n;  // warp-uniform
            float xf[TOK];
#pragma unroll
            for (int i = 0; i < TOK; ++i) xf[i] = raw_to_float(cur.e[i]);
            if (!full) {
#pragma unroll
                for (int i = 0; i < TOK; ++i)
                    if (t0 + i < 0) xf[i] = head[i];  // only in the first chunk
            }
            // p[j] = slot -j relative to this lane's first, from lane
            // l - ceil(j/TOK) of this chunk or (below lane 0) of the previous.
            float p[MAXW];
#pragma unroll
            for (int j = 1; j < MAXW; ++j) {
                if (j >= W) break;  // uniform across the warp
                const int src = lane - (j + TOK - 1) / TOK;
                const int e = (TOK - j % TOK) % TOK;
                const float vc = __shfl_sync(kFull, xf[e], src & 31);
                const float vp = __shfl_sync(kFull, prv[e], src & 31);
                p[j] = src >= 0 ? vc : vp;
            }
            Lanes<R, TOK> y;
#pragma unroll
            for (int i = 0; i < TOK; ++i) {
                float acc = bias;
#pragma unroll
                for (int d = MAXW - 1; d >= 0; --d) {
                    if (d >= W) continue;
                    acc = fmaf(wl[d], d <= i ? xf[i - d] : p[d - i], acc);
                }
                if (a.silu) acc = silu<E>(acc);
                y.e[i] = float_to_raw<E>(acc);
            }
            if (aligned_out && t0 >= 0 && t0 + TOK <= n) {
                *reinterpret_cast<uint4 *>(ov + k * CHUNK + TOK * lane) = y.v;
            } else {
#pragma unroll
                for (int i = 0; i < TOK; ++i)
                    if (t0 + i >= 0 && t0 + i < n) orow[t0 + i] = y.e[i];
            }
            if (st && (k + 1) * CHUNK - skew > n - L) {  // the chunk holds part of the last L
#pragma unroll
                for (int i = 0; i < TOK; ++i) {
                    const int t = t0 + i;
                    if (t >= 0 && t < n && t >= n - L)
                        st[static_cast<int64_t>(t - (n - L)) * a.s_k] = cur.e[i];
                }
            }
#pragma unroll
            for (int i = 0; i < TOK; ++i) prv[i] = xf[i];
        }
    }
}

// Prefill, any x layout: thread (b, c) walks sequence b's rows of channel c.
// prev[j-1] holds the input j rows back; lag-j weight wl[j] = weight[c][W-1-j].
template <typename E, int MAXW>
__global__ void __launch_bounds__(128) dense_fwd_generic(const __grid_constant__ DenseArgs a) {
    using R = typename RawOf<E>::T;
    const int b = blockIdx.x;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    pdl_wait();
    pdl_trigger();
    int q0, n;
    int64_t line;
    bool from;
    if (!sequence_setup(a, b, threadIdx.x == 0 && blockIdx.y == 0, q0, n, line, from)) return;
    if (c >= a.dim) return;

    const int W = a.W;
    const E *wp = static_cast<const E *>(a.w) + c * a.w_sc;
    float wl[MAXW];
#pragma unroll
    for (int j = 0; j < MAXW; ++j) wl[j] = j < W ? load_weight(wp + (W - 1 - j) * a.w_sk) : 0.f;
    const float bias = a.bias ? load_weight(static_cast<const E *>(a.bias) + c) : 0.f;

    R *st = a.st ? static_cast<R *>(a.st) + line * a.s_line + c * a.s_c : nullptr;
    const int L = a.L;
    float prev[MAXW - 1];
#pragma unroll
    for (int j = 1; j < MAXW; ++j)
        prev[j - 1] = (from && j < W) ? raw_to_float(st[(L - j) * a.s_k]) : 0.f;
    // Line entries that survive the call: new entry i = old entry n + i.
    if (st) {
        for (int i = 0; i < L && n + i < L; ++i) st[i * a.s_k] = from ? st[(n + i) * a.s_k] : R(0);
    }

    const R *x = static_cast<const R *>(a.x) + static_cast<int64_t>(q0) * a.x_st +
                 static_cast<int64_t>(c) * a.x_sc;
    R *out = static_cast<R *>(a.out) + static_cast<int64_t>(q0) * a.x_st +
             static_cast<int64_t>(c) * a.x_sc;
    for (int t = 0; t < n; ++t) {
        const R xr = x[static_cast<int64_t>(t) * a.x_st];
        const float xf = raw_to_float(xr);
        float acc = bias;
#pragma unroll
        for (int j = MAXW - 1; j >= 1; --j)
            if (j < W) acc = fmaf(wl[j], prev[j - 1], acc);
        acc = fmaf(wl[0], xf, acc);
#pragma unroll
        for (int j = MAXW - 2; j >= 1; --j) prev[j] = prev[j - 1];
        prev[0] = xf;
        if (a.silu) acc = silu<E>(acc);
        out[static_cast<int64_t>(t) * a.x_st] = float_to_raw<E>(acc);
        if (st && t >= n - L) st[(t - (n - L)) * a.s_k] = xr;
    }
}


// Decode: thread (b, j) updates channels c .. c+VEC-1 of sequence b, 4 bytes
// of channels (2 bf16 or 1 fp32): many threads with little serial work each,
// since one decode step is bound by memory latency, not bandwidth.  Each
// thread loads its channels' weights before the wait for the preceding
// kernel (they are constant; staging the block's weights through shared
// memory instead cost 1.2 us per launch).  Every line entry the update needs
// is read before the first write, so the line costs one memory round trip.  Line access by
// layout (MODE = DenseArgs::st_mode): 0 single elements; 1 one VEC-element
// vector per entry; 2 the block's whole run of lines (VEC*L contiguous
// elements per thread) staged through shared memory with 16-byte copies,
// updated there by each thread for its own channels, and copied back.
template <typename E, int VEC, int MAXW, int LMAX, int MODE>
__global__ void __launch_bounds__(128) dense_update(const __grid_constant__ DenseArgs a) {
    using R = typename RawOf<E>::T;
    using LV = Lanes<R, VEC>;
    extern __shared__ uint4 smem16[];
    const int b = blockIdx.x;
    const int c0 = blockIdx.y * blockDim.x * VEC;  // first channel of the block
    const int nch = min(static_cast<int>(blockDim.x) * VEC, a.dim - c0);
    const int c = c0 + threadIdx.x * VEC;
    const bool active = c < a.dim;
    const int L = a.L, W = a.W;

    float wt[MAXW][VEC];
    float acc[VEC];
    if (active) {
        load_taps<E, VEC, MAXW>(a, c, wt);
        load_bias<E, VEC>(a, c, acc);
    }
    // While the preceding kernel drains: the x pack and, from a speculative
    // read of the line index (L2-only, range-checked), the thread's line
    // entries into L2.  A stale index costs a useless prefetch only.
    if (active) {
        prefetch_l2(static_cast<const R *>(a.x) + static_cast<int64_t>(b) * a.x_st +
                    static_cast<int64_t>(c) * a.x_sc);
        const int64_t ls = a.lines ? __ldcg(a.lines + b) : b;
        if (ls >= 0 && ls < a.num_lines && !(a.lines && ls == a.pad)) {
            const R *sp = static_cast<const R *>(a.st) + ls * a.s_line +
                          static_cast<int64_t>(c) * a.s_c;
            for (int i = 0; i < L; ++i) prefetch_l2(sp + i * a.s_k);
        }
    }
    if (threadIdx.x == 0 && a.seqlens) prefetch_l2(a.seqlens + b);
    pdl_wait();
    pdl_trigger();
    const int64_t line = a.lines ? __ldg(a.lines + b) : b;
    if (a.lines && line == a.pad) return;
    if (line < 0 || line >= a.num_lines) {
        if (threadIdx.x == 0 && blockIdx.y == 0) flag(a.err, SCONV_EFLAG_SLOT);
        return;
    }
    // x (issued before the line, which waits on the index): plain loads,
    // since with out == x this kernel writes it.
    R xr[VEC];
    if (active) {
        const R *xp = static_cast<const R *>(a.x) + static_cast<int64_t>(b) * a.x_st +
                      static_cast<int64_t>(c) * a.x_sc;
        if constexpr (VEC > 1) {
            LV xin;
            xin.v = *reinterpret_cast<const typename RawVec<VEC * sizeof(R)>::T *>(xp);
#pragma unroll
            for (int v = 0; v < VEC; ++v) xr[v] = xin.e[v];
        } else {
            xr[0] = *xp;
        }
    }
    const bool ring = a.seqlens != nullptr;
    const int64_t s = ring ? __ldg(a.seqlens + b) : 0;
    R *st = static_cast<R *>(a.st) + line * a.s_line + static_cast<int64_t>(c) * a.s_c;

    // MODE 2: stage this block's contiguous run of lines.
    uint4 *run16 = smem16;
    R *mine = reinterpret_cast<R *>(run16) + threadIdx.x * VEC * L;
    int n16 = 0;
    uint4 *grun = nullptr;
    if constexpr (MODE == 2) {
        n16 = nch * L * static_cast<int>(sizeof(R)) / 16;
        grun = reinterpret_cast<uint4 *>(static_cast<R *>(a.st) + line * a.s_line +
                                         static_cast<int64_t>(c0) * L);
        for (int j = threadIdx.x; j < n16; j += blockDim.x) run16[j] = grun[j];
    }
    __syncthreads();  // the block's lines staged (MODE 2)

    // Entry i of the thread's VEC channels.
    auto get = [&](int64_t i, R (&e)[VEC]) {
        if constexpr (MODE == 1) {
            LV p;
            p.v = *reinterpret_cast<const typename RawVec<VEC * sizeof(R)>::T *>(st + i * a.s_k);
#pragma unroll
            for (int v = 0; v < VEC; ++v) e[v] = p.e[v];
        } else if constexpr (MODE == 2) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) e[v] = mine[v * L + i];
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) e[v] = st[v * a.s_c + i * a.s_k];
        }
    };
    auto put = [&](int64_t i, const R (&e)[VEC]) {
        if constexpr (MODE == 1) {
            LV p;
#pragma unroll
            for (int v = 0; v < VEC; ++v) p.e[v] = e[v];
            *reinterpret_cast<typename RawVec<VEC * sizeof(R)>::T *>(st + i * a.s_k) = p.v;
        } else if constexpr (MODE == 2) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) mine[v * L + i] = e[v];
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) st[v * a.s_c + i * a.s_k] = e[v];
        }
    };

    if (active) {
        // The W-1 taps before the token, by tap slot, and (shifted line) the
        // entries 1..L-1 that move down one place.
        R tap[MAXW - 1][VEC];
#pragma unroll
        for (int kk = 0; kk < MAXW - 1; ++kk) {
            const int k = kk - (MAXW - W);
            if (k < 0) continue;
            int64_t i = L - (W - 1) + k;
            if (ring) {
                i = (s - (W - 1) + k) % L;
                if (i < 0) i += L;
            }
            get(i, tap[kk]);
        }
        R keep[LMAX - 1][VEC];
        if (!ring) {
#pragma unroll
            for (int i = 0; i < LMAX - 1; ++i)
                if (i + 1 < L) get(i + 1, keep[i]);
        }

#pragma unroll
        for (int v = 0; v < VEC; ++v) {
#pragma unroll
            for (int kk = 0; kk < MAXW - 1; ++kk) {
                const int k = kk - (MAXW - W);
                if (k >= 0) acc[v] = fmaf(wt[kk][v], raw_to_float(tap[kk][v]), acc[v]);
            }
            acc[v] = fmaf(wt[MAXW - 1][v], raw_to_float(xr[v]), acc[v]);
            if (a.silu) acc[v] = silu<E>(acc[v]);
        }

        if (ring) {
            int64_t i = s % L;
            if (i < 0) i += L;
            put(i, xr);
        } else {
#pragma unroll
            for (int i = 0; i < LMAX - 1; ++i)
                if (i + 1 < L) put(i, keep[i]);
            put(L - 1, xr);
        }
        R *op = static_cast<R *>(a.out) + static_cast<int64_t>(b) * a.x_st +
                static_cast<int64_t>(c) * a.x_sc;
        if constexpr (VEC > 1) {
            LV o;
#pragma unroll
            for (int v = 0; v < VEC; ++v) o.e[v] = float_to_raw<E>(acc[v]);
            *reinterpret_cast<typename RawVec<VEC * sizeof(R)>::T *>(op) = o.v;
        } else {
            *op = float_to_raw<E>(acc[0]);
        }
    }
    if constexpr (MODE == 2) {
        __syncthreads();
        for (int j = threadIdx.x; j < n16; j += blockDim.x) grun[j] = run16[j];
    }
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 148;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            n = v;
        else
            n = 148;
    }
    return n;
}

// Packs per block: the widest column (up to 8 packs, 128 bytes of a row)
// that still gives at least 1.5 blocks per SM.  Every block streams a whole
// column, so wide columns read whole 128-byte lines and keep the DRAM
// accesses of a row together, while a few long sequences need narrower
// columns to spread their channels over the chip.
int pick_pp(int batch, int packs) {
    const int64_t want = 3LL * sm_count() / 2;
    int pp = 8;
    while (pp > 1 && pp > packs) pp /= 2;
    for (; pp > 1; pp /= 2)
        if (static_cast<int64_t>(batch) * ((packs + pp - 1) / pp) >= want) return pp;
    return 1;
}

template <typename E, int PP, int WT, int THREADS, int STAGES>
cudaError_t launch_tile_pp(const DenseArgs &a, const CUtensorMap &map, int packs,
                           cudaStream_t stream) {
    constexpr int kSmem = TileLayout<PP, WT, THREADS, STAGES>::smem;
    auto kernel = dense_fwd_tile<E, PP, WT, THREADS, STAGES>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [&] {
        attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    });
    if (attr != cudaSuccess) return attr;
    const int ncb = (packs + PP - 1) / PP;
    return launch_pdl(kernel, dim3(static_cast<unsigned>(static_cast<int64_t>(a.batch) * ncb)),
                      dim3(THREADS), static_cast<size_t>(kSmem), stream, a, map, ncb);
}

template <typename E, int PP, int WT>
cudaError_t launch_tile_s(const DenseArgs &a, const CUtensorMap &map, int packs,
                          cudaStream_t stream) {
    // Several waves: 3 resident blocks per SM is what registers allow.
    const int64_t blocks = static_cast<int64_t>(a.batch) * ((packs + PP - 1) / PP);
    if (blocks >= 2LL * 3 * sm_count())
        return launch_tile_pp<E, PP, WT, kTileThreads, kStagesFew>(a, map, packs, stream);
    return launch_tile_pp<E, PP, WT, kTileThreads, kStagesMany>(a, map, packs, stream);
}

template <typename E, int WT>
cudaError_t launch_tile_w(const DenseArgs &a, const CUtensorMap &map, int packs, int pp,
                          cudaStream_t stream) {
    switch (pp) {
        case 8: return launch_tile_s<E, 8, WT>(a, map, packs, stream);
        case 4: return launch_tile_s<E, 4, WT>(a, map, packs, stream);
        case 2: return launch_tile_s<E, 2, WT>(a, map, packs, stream);
        default: return launch_tile_s<E, 1, WT>(a, map, packs, stream);
    }
}

// The tensor map of x for a column of pp packs: rows of dim channels (a
// stride of x_st elements), boxes of pp packs x min(TT, 256) rows.  Rows
// past T and channels past dim arrive as zeros.  False when the driver
// offers no encoder or rejects the layout.
template <typename E>
bool encode_tile_map(const DenseArgs &a, int pp, CUtensorMap &map) {
    constexpr int VEC = 16 / sizeof(E);
    constexpr int64_t e = sizeof(E);
    if (tma::encode_fn() == nullptr) return false;
    const int tt = kTileThreads / pp * kRowsPerThread;
    // Tile row coordinates (up to T + TT) are 32-bit copy coordinates.
    if (static_cast<int64_t>(a.T) + tt >= (1ll << 31)) return false;
    const cuuint64_t dim[2] = {static_cast<cuuint64_t>(a.dim),
                               static_cast<cuuint64_t>(a.T > 1 ? a.T : 1)};
    // With one row the stride is never used; any legal value will do.
    const int64_t row = a.T > 1 ? a.x_st * e : (a.dim * e + 15) / 16 * 16;
    const cuuint64_t stride[1] = {static_cast<cuuint64_t>(row)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(pp * VEC),
                               static_cast<cuuint32_t>(tt > 256 ? 256 : tt)};
    const cuuint32_t elem[2] = {1, 1};
    const CUtensorMapDataType type =
        e == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return tma::encode_fn()(&map, type, 2, const_cast<void *>(a.x), dim, stride, box, elem,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tiled prefill; `used` false (nothing launched) when x has no tensor
// map, for the caller to take another kernel.
template <typename E>
cudaError_t launch_tile(const DenseArgs &a, cudaStream_t stream, bool &used) {
    constexpr int VEC = 16 / sizeof(E);
    const int packs = a.dim / VEC;
    const int pp = pick_pp(a.batch, packs);
    CUtensorMap map;
    used = encode_tile_map<E>(a, pp, map);
    if (!used) return cudaSuccess;
    switch (a.W) {
        case 2: return launch_tile_w<E, 2>(a, map, packs, pp, stream);
        case 3: return launch_tile_w<E, 3>(a, map, packs, pp, stream);
        case 4: return launch_tile_w<E, 4>(a, map, packs, pp, stream);
        default: return launch_tile_w<E, 8>(a, map, packs, pp, stream);
    }
}

template <typename E, int MAXW>
cudaError_t launch_fwd_t(const DenseArgs &a, bool vec, cudaStream_t stream) {
    if (vec) {
        bool used = false;
        const cudaError_t e = launch_tile<E>(a, stream, used);
        if (used) return e;
    }
    if (a.x_st == 1 && a.T > 1 && (reinterpret_cast<uintptr_t>(a.x) & 15u) == 0) {
        // channel-major: a warp per (sequence, channel)
        const int64_t warps = static_cast<int64_t>(a.batch) * a.dim;
        return launch_pdl(dense_fwd_cm<E, MAXW>, dim3(static_cast<unsigned>((warps + 7) / 8)),
                          dim3(256), 0, stream, a);
    }
    return launch_pdl(dense_fwd_generic<E, MAXW>, dim3(a.batch, (a.dim + 127) / 128), dim3(128),
                      0, stream, a);
}

// Decode threads own 4 bytes of channels (2 bf16 or 1 fp32) on the vector
// path, one channel otherwise.
template <typename E, int MAXW, int LMAX>
cudaError_t launch_update_l(const DenseArgs &a, bool vec, cudaStream_t stream) {
    constexpr int VEC = 4 / sizeof(E);
    const int v = vec ? VEC : 1;
    const int per_block = 128 * v;
    const dim3 grid(a.T, (a.dim + per_block - 1) / per_block);
    const int nch = a.dim < per_block ? a.dim : per_block;
    size_t smem = 0;
    if (!vec)
        return launch_pdl(dense_update<E, 1, MAXW, LMAX, 0>, grid, dim3(128), smem, stream, a);
    switch (a.st_mode) {
        case 1:
            return launch_pdl(dense_update<E, VEC, MAXW, LMAX, 1>, grid, dim3(128), smem, stream, a);
        case 2:
            smem += static_cast<size_t>(nch) * a.L * sizeof(E);
            return launch_pdl(dense_update<E, VEC, MAXW, LMAX, 2>, grid, dim3(128), smem, stream, a);
        default:
            return launch_pdl(dense_update<E, VEC, MAXW, LMAX, 0>, grid, dim3(128), smem, stream, a);
    }
}

template <typename E, int MAXW>
cudaError_t launch_update_t(const DenseArgs &a, bool vec, cudaStream_t stream) {
    return a.L <= 4 ? launch_update_l<E, MAXW, 4>(a, vec, stream)
                    : launch_update_l<E, MAXW, kMaxL>(a, vec, stream);
}

}  // namespace

cudaError_t launch_dense_fwd(const DenseArgs &a, bool bf16_data, bool vec, cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    if (bf16_data)
        return a.W <= 4 ? launch_fwd_t<bf16, 4>(a, vec, stream) : launch_fwd_t<bf16, 8>(a, vec, stream);
    return a.W <= 4 ? launch_fwd_t<float, 4>(a, vec, stream) : launch_fwd_t<float, 8>(a, vec, stream);
}

cudaError_t launch_dense_update(const DenseArgs &a, bool bf16_data, bool vec,
                                cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    if (bf16_data)
        return a.W <= 4 ? launch_update_t<bf16, 4>(a, vec, stream)
                        : launch_update_t<bf16, 8>(a, vec, stream);
    return a.W <= 4 ? launch_update_t<float, 4>(a, vec, stream)
                    : launch_update_t<float, 8>(a, vec, stream);
}

}  // namespace sconv
