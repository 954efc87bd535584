// fused_tma.cu -- the prefill form of the fused insert + causal conv1d
// ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv) with its x tiles
// and per-token metadata staged in shared memory by the Tensor Memory
// Accelerator, for sm_100a.
//
// Tiling.  A tile is kBT = 32 consecutive tokens x 512 bytes of a row (256
// bf16 or 128 fp32 channels, kBC<E>).  One thread of each block issues, per
// tile,
//   * a 2-D tensor copy of x rows [t0 - (W-1), t0 + 32) x [c0, c0 + kBC<E>)
//     (the W-1 halo rows before the tile included; rows before 0 and past T
//     and channels past C arrive as zeros), and
//   * four 1-D tensor copies of the tile's positions, slot_mapping, seq_idx
//     and query_start,
// all completing on one mbarrier.  Tiles flow through a ring of STAGES
// shared-memory stages, so up to STAGES-1 tiles are in flight while one is
// computed: the memory system sees a steady stream of bulk copies whatever
// the register budget of the compute threads.  The grid is persistent, one
// block per resident slot (SMs x blocks per SM).  Work units are (token
// tile, channel block) pairs numbered token-tile major, u = tile * ncb + cb,
// and block b takes u = b, b + grid, b + 2 grid, ...: at any moment the grid
// works on one contiguous run of units, a compact band of x, out and the
// cache rows, and every block ends within one unit of the others.  DRAM
// serves that band far faster than one scattered spot per block (chunked
// prefill 82.2 -> 72.3 us, long prefill 611 -> 530 us, against equal
// contiguous shares of the units in channel-block-major order).  A block's
// channel block changes from unit to unit; when it does, the block reloads
// its weights (a few lines, L1-resident) or, for bf16 W > 4 and fp32 W > 5,
// copies them from the shared-memory set it unpacked at entry.
//
// Compute.  Eight warps per block; warp g owns tokens 4g..4g+3 of the tile
// and lane l the 16-byte pack l of the tile's row (8 bf16 or 4 fp32
// channels).  W, the tap count 1..8, is a template parameter.  Lanes
// 0..3 classify the warp's four tokens (ordinary, PAD, or needing cache
// taps / out of range) and compute their cache insert offsets once; when all
// four are ordinary -- nearly always in prefill -- one straight-line block
// convolves them from the W+3 shared-memory rows they need (16-byte loads,
// conflict-free: a warp reads one contiguous 512-byte row).  When the
// other tokens of a warp are the opening tokens of one request, the
// request's last W-1 cached rows replace the x rows before it in the
// warp's register window, in one round of loads, and the same block
// convolves them.  Otherwise each token takes the general path, where taps
// that precede the token's request come from the cache through the block
// table, one after another.  Outputs and cache inserts are 16-byte stores
// straight to global memory.
//
// Every wait on an mbarrier is bounded; a block whose copies do not arrive
// in time sets SCONV_EFLAG_TIMEOUT, waits (bounded) for its other copies and
// returns without writing anything for that tile.
#include <atomic>

#include "common.cuh"
#include "fused_common.cuh"
#include "sconv.h"
#include "tma.cuh"

namespace sconv {
namespace {

using namespace tma;

template <typename E>
constexpr int kBC = 512 / static_cast<int>(sizeof(E));  // channels per tile
constexpr int kBT = 32;            // tokens per tile
constexpr int kThreads = 256;      // 8 warps
constexpr int kTokPerWarp = kBT / (kThreads / 32);  // 4
constexpr int kMetaBytes = kBT * (8 + 8 + 4 + 4);   // positions, slots, seq_idx, query_start

// A stage: the x rows, then the tile's metadata -- positions, slots,
// seq_idx and query_start, or, with TAPS, the slots and the tokens' rows of
// the resolved tap table (W-1 int64 each).  Every part starts on a 128-byte
// boundary.
template <int W, bool TAPS = false>
struct Layout {
    static constexpr int rows = kBT + W - 1;
    static constexpr int x_bytes = rows * 512;  // multiple of 512: TMA destinations stay 128-B aligned
    static constexpr int meta = TAPS ? kBT * 8 * W : kMetaBytes;
    static constexpr int stage = x_bytes + meta;
};

template <int W, int STAGES, bool TAPS = false>
constexpr int kStages_smem() {
    return STAGES * Layout<W, TAPS>::stage + 2 * STAGES * 8;
}

// Shared memory for cached weights: room for ncache * W 512-byte lag rows
// that still leaves two blocks per SM at every W.  Reloading (and, for bf16,
// re-pairing) the weights at each channel-block switch is cheap up to W = 4
// (bf16) or 5 (fp32) and costs more than the shared-memory copy beyond (A/B
// on the chunked prefill shape, us: bf16 W 4 / 5 / 6 / 8: reload 72.4 /
// 96.1 / 139.0 / 123.4, cached 76.0 / 75.9 / 82.0 / 93.0; fp32 W 4 / 6 / 8:
// reload 149.2 / 185.5 / 211.3, cached 153.6 / 148.6 / 155.5).
constexpr int kWeightCacheBytes = 24 * 1024;
template <typename E, int W>
constexpr bool kCachesWeights = W > (sizeof(E) == 2 ? 4 : 5);

struct TmaMaps {
    CUtensorMap x, pos, slot, sid, qs, tab;  // tab: the resolved tap table (TAPS)
};

template <typename E>
using PackOf = Pack<E, 16 / sizeof(E)>;

// acc += w * tap for one 8-channel pack: eight fp32-accumulating FMAs that
// take bf16 operands directly (the product of two bf16 values is exact in
// fp32, so this equals widening both and one fmaf, bit for bit).  w holds
// the pack's weights for one lag as four bf16 pairs.
__device__ __forceinline__ void fma_pack(float (&acc)[8], const uint32_t (&w)[4],
                                         const Pack<bf16, 8> &tap) {
    const uint32_t q[4] = {tap.u.x, tap.u.y, tap.u.z, tap.u.w};
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

// The pack's weights by lag (lag d multiplies position pos - d, weight
// column W-1-d).  With a dense [C, W] weight the pack's VEC*W elements are
// contiguous and 16-byte aligned: W vector loads.
template <typename E, int W>
struct LagWeights;

template <int W>
struct LagWeights<bf16, W> {
    uint32_t w[W][4];  // bf16 pairs, channel 2i in the low half
    __device__ __forceinline__ void load(const FusedArgs &a, int c) {
        const unsigned short *wp = static_cast<const unsigned short *>(a.w);
        unsigned short e[8][W];
        if (a.w_vec) {
            union {
                uint4 u[W];
                unsigned short h[8 * W];
            } raw;
            const uint4 *p = reinterpret_cast<const uint4 *>(wp + static_cast<int64_t>(c) * W);
#pragma unroll
            for (int q = 0; q < W; ++q) raw.u[q] = __ldg(p + q);
#pragma unroll
            for (int v = 0; v < 8; ++v)
#pragma unroll
                for (int d = 0; d < W; ++d) e[v][d] = raw.h[v * W + W - 1 - d];
        } else {
#pragma unroll
            for (int v = 0; v < 8; ++v)
#pragma unroll
                for (int d = 0; d < W; ++d)
                    e[v][d] = __ldg(wp + static_cast<int64_t>(c + v) * a.w_sc +
                                    static_cast<int64_t>(W - 1 - d) * a.w_sk);
        }
#pragma unroll
        for (int d = 0; d < W; ++d)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[d][i] = static_cast<uint32_t>(e[2 * i][d]) |
                          (static_cast<uint32_t>(e[2 * i + 1][d]) << 16);
    }
    __device__ __forceinline__ void fma(float (&acc)[8], int d, const Pack<bf16, 8> &tap) const {
        fma_pack(acc, w[d], tap);
    }
    // Lag d of this lane at wc[d * 32 + lane]: conflict-free 16-byte accesses.
    __device__ __forceinline__ void to_smem(uint4 *wc, int lane) const {
#pragma unroll
        for (int d = 0; d < W; ++d) wc[d * 32 + lane] = make_uint4(w[d][0], w[d][1], w[d][2], w[d][3]);
    }
    __device__ __forceinline__ void from_smem(const uint4 *wc, int lane) {
#pragma unroll
        for (int d = 0; d < W; ++d) {
            const uint4 q = wc[d * 32 + lane];
            w[d][0] = q.x;
            w[d][1] = q.y;
            w[d][2] = q.z;
            w[d][3] = q.w;
        }
    }
};

template <int W>
struct LagWeights<float, W> {
    float w[W][4];
    __device__ __forceinline__ void load(const FusedArgs &a, int c) {
        const float *wp = static_cast<const float *>(a.w);
        if (a.w_vec) {
            union {
                uint4 u[W];
                float f[4 * W];
            } raw;
            const uint4 *p = reinterpret_cast<const uint4 *>(wp + static_cast<int64_t>(c) * W);
#pragma unroll
            for (int q = 0; q < W; ++q) raw.u[q] = __ldg(p + q);
#pragma unroll
            for (int v = 0; v < 4; ++v)
#pragma unroll
                for (int d = 0; d < W; ++d) w[d][v] = raw.f[v * W + W - 1 - d];
        } else {
#pragma unroll
            for (int v = 0; v < 4; ++v)
#pragma unroll
                for (int d = 0; d < W; ++d)
                    w[d][v] = __ldg(wp + static_cast<int64_t>(c + v) * a.w_sc +
                                    static_cast<int64_t>(W - 1 - d) * a.w_sk);
        }
    }
    __device__ __forceinline__ void fma(float (&acc)[4], int d, const Pack<float, 4> &tap) const {
        float t[4];
        tap.to_float(t);
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[v] = fmaf(w[d][v], t[v], acc[v]);
    }
    __device__ __forceinline__ void to_smem(uint4 *wc, int lane) const {
#pragma unroll
        for (int d = 0; d < W; ++d)
            wc[d * 32 + lane] = make_uint4(__float_as_uint(w[d][0]), __float_as_uint(w[d][1]),
                                           __float_as_uint(w[d][2]), __float_as_uint(w[d][3]));
    }
    __device__ __forceinline__ void from_smem(const uint4 *wc, int lane) {
#pragma unroll
        for (int d = 0; d < W; ++d) {
            const uint4 q = wc[d * 32 + lane];
            w[d][0] = __uint_as_float(q.x);
            w[d][1] = __uint_as_float(q.y);
            w[d][2] = __uint_as_float(q.z);
            w[d][3] = __uint_as_float(q.w);
        }
    }
};

// SCONV_EFLAG_* bits of a non-PAD token of the resolved-tap form from its
// table row (W-1 entries, lag d at row[d-1]) and slot: the bits the token
// form (sconv_fused_taps) reports for the same token -- the row's failure
// codes, SCONV_EFLAG_BLOCK for a slot past the cache or an entry that is no
// valid code, SCONV_EFLAG_QUERY_START for an x row before the call's first,
// and for a slot out of range SCONV_EFLAG_SLOT with the row's request,
// query-start and position bits.
template <int W>
__device__ __forceinline__ unsigned tab_flags(const int64_t *row, int t, int64_t slot,
                                              int64_t slots_total) {
    unsigned f = 0;
#pragma unroll
    for (int d = 1; d < W; ++d) {
        const int64_t e = row[d - 1];
        if (e >= 0) {
            if (e >= slots_total) f |= SCONV_EFLAG_BLOCK;
        } else if (e == SCONV_TAP_X) {
            if (t - d < 0) f |= SCONV_EFLAG_QUERY_START;
        } else if (e != SCONV_TAP_ZERO) {
            const unsigned bits =
                e <= -256 ? static_cast<unsigned>((~static_cast<uint64_t>(e) + 1) >> 8) & 0x3fu
                          : 0u;
            f |= bits ? bits : SCONV_EFLAG_BLOCK;
        }
    }
    if (slot < 0 || slot >= slots_total)
        f = SCONV_EFLAG_SLOT |
            (f & (SCONV_EFLAG_REQUEST | SCONV_EFLAG_QUERY_START | SCONV_EFLAG_POSITION));
    return f;
}

// The pack lane l works on in channel block cb (clamped to the last pack
// for lanes past C, which compute but store nothing).
__device__ __forceinline__ int cb_pack(int cb, int l, int nv) {
    const int p = cb * 32 + l;
    return p < nv ? p : nv - 1;
}

// What a warp's lane u (< kTokPerWarp) knows about token u of its group.
enum : int { kSkip = 0, kFast = 1, kSlow = 2 };

template <typename E, int W, int STAGES, bool SILU, bool RESID, bool TAPS = false>
__global__ void __launch_bounds__(kThreads, STAGES <= 3 ? 3 : 2)
fused_tma_kernel(const __grid_constant__ FusedArgs a, const __grid_constant__ TmaMaps maps,
                 int ncache) {
    using L = Layout<W, TAPS>;
    using P = PackOf<E>;
    constexpr int VEC = 16 / static_cast<int>(sizeof(E));
    constexpr int BC = kBC<E>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * L::stage);
    uint64_t *empty = full + STAGES;
    uint4 *wcache = reinterpret_cast<uint4 *>(empty + STAGES);  // ncache x W x 32 lanes

    // This block's units: u = b0, b0 + gstride, ... below ntiles * ncb.
    const int ntiles = (a.T + kBT - 1) / kBT;
    const int ncb = (a.C + BC - 1) / BC;
    const int64_t units = static_cast<int64_t>(ntiles) * ncb;
    const int64_t gstride = gridDim.x;
    const int64_t b0 = blockIdx.x;
    const int my = b0 < units ? static_cast<int>((units - 1 - b0) / gstride + 1) : 0;
    if (my <= 0) return;  // whole block

    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kThreads / 32);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();  // inputs may come from the previous kernel in the stream
    pdl_trigger();

    int issued = 0;  // tiles issued so far (meaningful in thread 0, the producer)
    auto issue = [&](int k) {
        ++issued;
        const int s = k % STAGES;
        unsigned char *st = smem + s * L::stage;
        const int64_t u = b0 + k * gstride;
        const int c0 = static_cast<int>(u % ncb) * BC;
        const int t0 = static_cast<int>(u / ncb) * kBT;
        mbar_expect_tx(&full[s], L::stage);
        copy_2d(st, &maps.x, c0, t0 - (W - 1), &full[s]);
        if constexpr (TAPS) {
            copy_1d(st + L::x_bytes, &maps.slot, t0, &full[s]);
            if constexpr (W > 1) copy_1d(st + L::x_bytes + kBT * 8, &maps.tab, t0 * (W - 1), &full[s]);
        } else {
            copy_1d(st + L::x_bytes, &maps.pos, t0, &full[s]);
            copy_1d(st + L::x_bytes + kBT * 8, &maps.slot, t0, &full[s]);
            copy_1d(st + L::x_bytes + kBT * 16, &maps.sid, t0, &full[s]);
            copy_1d(st + L::x_bytes + kBT * 20, &maps.qs, t0, &full[s]);
        }
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < STAGES && k < my; ++k) issue(k);

    const int lane_id = threadIdx.x & 31;
    // A block's channel block repeats with period ncache (ncache * gstride
    // is a multiple of ncb); when the host found room, the weights of those
    // channel blocks are unpacked once into shared memory, so a switch costs
    // W shared-memory loads instead of W global loads and the unpacking.
    if (kCachesWeights<E, W> && ncache > 0) {
        for (int j = threadIdx.x >> 5; j < ncache; j += kThreads / 32) {
            const int cbj = static_cast<int>((b0 + j * gstride) % ncb);
            const int pj = cb_pack(cbj, lane_id, a.C / VEC);
            LagWeights<E, W> t;
            t.load(a, pj * VEC);
            t.to_smem(wcache + j * W * 32, lane_id);
        }
        __syncthreads();
    }
    const int i0 = (threadIdx.x >> 5) * kTokPerWarp;
    const int nv = a.C / VEC;
    const int64_t slots_total = a.num_blocks * a.N;
    int cur_cb = -1;
    bool active = false;
    int c = 0;
    int64_t lane = 0;
    LagWeights<E, W> wr;
    bool alive = true;
    int next = 0;  // the next tile this thread waits for

    for (int k = 0; k < my; ++k) {
        next = k;
        const int s = k % STAGES;
        const int64_t u = b0 + k * gstride;
        const int cb = static_cast<int>(u % ncb);
        const int t0 = static_cast<int>(u / ncb) * kBT;
        if (cb != cur_cb) {  // a new channel block: its taps and cache lanes
            cur_cb = cb;
            active = cb * 32 + lane_id < nv;
            c = cb_pack(cb, lane_id, nv) * VEC;
            const int h = c / a.ws;
            lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
            if (kCachesWeights<E, W> && ncache > 0)
                wr.from_smem(wcache + (k % ncache) * W * 32, lane_id);
            else
                wr.load(a, c);
        }
        if (!mbar_wait(&full[s], (k / STAGES) & 1)) {  // copies did not arrive in time
            if (a.err && lane_id == 0) atomicOr(a.err, static_cast<int>(SCONV_EFLAG_TIMEOUT));
            alive = false;
            break;
        }
        const unsigned char *st = smem + s * L::stage;
        const P *xs = reinterpret_cast<const P *>(st) + lane_id;  // row r at xs[r * 32]
        const int64_t *mpos = reinterpret_cast<const int64_t *>(st + L::x_bytes);
        const int64_t *mslot = TAPS ? mpos : mpos + kBT;
        const int32_t *msid = reinterpret_cast<const int32_t *>(st + L::x_bytes + kBT * 16);
        const int32_t *mqs = msid + kBT;
        const int64_t *mtab = mslot + kBT;  // TAPS: token i's table row at mtab[i * (W-1)]

        // Lanes 0..3 classify the group's tokens and address their inserts.
        int code = kSkip;
        int64_t ins = 0;
        if (TAPS && lane_id < kTokPerWarp) {
            // Ordinary: every tap an x row of this call; otherwise the
            // general path (cache taps, zero taps or an index error).
            const int i = i0 + lane_id;
            const int t = t0 + i;
            const int64_t slot = mslot[i];
            if (t < a.T && slot != -1) {
                const int64_t *row = mtab + i * (W - 1);
                bool all_x = true;
#pragma unroll
                for (int d = 1; d < W; ++d) all_x = all_x && row[d - 1] == SCONV_TAP_X;
                const bool bad = tab_flags<W>(row, t, slot, slots_total) != 0;
                code = (!bad && all_x) ? kFast : kSlow;
                if (slot >= 0 && slot < slots_total) {
                    int64_t blk, off;
                    split_n(a, slot, a.slots32 != 0, blk, off);
                    ins = blk * a.cs0 + off * a.cs2;
                }
            }
        } else if (!TAPS && lane_id < kTokPerWarp) {
            const int i = i0 + lane_id;
            const int t = t0 + i;
            const int64_t slot = mslot[i];
            if (t < a.T && slot != -1) {
                const int64_t pos = mpos[i];
                const int req = msid[i];
                const int q0 = mqs[i];
                const bool bad = slot < 0 || slot >= slots_total || req < 0 ||
                                 req >= a.num_reqs || q0 < 0 || q0 > t || pos < 0;
                code = (!bad && t - q0 >= W - 1) ? kFast : kSlow;
                if (!bad) {
                    int64_t blk, off;
                    split_n(a, slot, a.slots32 != 0, blk, off);
                    ins = blk * a.cs0 + off * a.cs2;
                }
            }
        }
        const unsigned fast_mask = __ballot_sync(0xffffffffu, code == kFast);

        // Shared-memory row r holds x row t0 - (W-1) + r; token i at lag d
        // reads row i + (W-1) - d.
        P rows[kTokPerWarp + W - 1];
#pragma unroll
        for (int r = 0; r < kTokPerWarp + W - 1; ++r) rows[r] = xs[(i0 + r) * 32];

        E *out = static_cast<E *>(a.out);
        E *cache = static_cast<E *>(a.cache);
        if ((fast_mask & 0xfu) == 0xfu) {
            // The common case: four ordinary tokens, straight-line code.
#pragma unroll
            for (int uu = 0; uu < kTokPerWarp; ++uu) {
                float acc[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
#pragma unroll
                for (int d = W - 1; d >= 0; --d) wr.fma(acc, d, rows[uu + W - 1 - d]);
                const int64_t ins_u = __shfl_sync(0xffffffffu, ins, uu);
                float xc[VEC];
                rows[uu + W - 1].to_float(xc);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    float y = acc[v];
                    if (SILU) y = silu<E>(y);
                    if (RESID) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
                    acc[v] = y;
                }
                P o;
                o.from_float(acc);
                if (active) {
                    o.store(out + static_cast<int64_t>(t0 + i0 + uu) * a.out_rs + c);
                    rows[uu + W - 1].store(cache + ins_u + lane);
                }
            }
        } else {
            // Staged route: when the group's slow tokens all open one
            // request (first row q0g, its first position p0g >= W-1, the
            // positions consecutive, every index valid), their cache taps
            // are the request's last W-1 cached rows.  Those rows replace,
            // in the register window, the x rows before q0g -- once the
            // group's tokens of the previous request are done with them --
            // in one round of loads, and the request's tokens then take the
            // straight-line path.  Otherwise every token takes the general
            // path below.
            bool staged = false;
            int split = 0, q0g = 0, reqg = 0;
            int64_t p0g = 0;
            if constexpr (!TAPS) {
                bool ok = true, any = false;
#pragma unroll
                for (int uu = 0; uu < kTokPerWarp; ++uu) {
                    if (__shfl_sync(0xffffffffu, code, uu) != kSlow) continue;
                    const int i = i0 + uu;
                    const int t = t0 + i;
                    const int64_t slot = mslot[i];
                    const int64_t pos = mpos[i];
                    const int req = msid[i];
                    const int q0 = mqs[i];
                    if (slot < 0 || slot >= slots_total || req < 0 || req >= a.num_reqs ||
                        q0 < 0 || q0 > t || pos < 0)
                        ok = false;
                    if (!any) {
                        any = true;
                        q0g = q0;
                        reqg = req;
                        p0g = pos - (t - q0);
                    } else if (q0 != q0g || req != reqg || pos - (t - q0) != p0g) {
                        ok = false;
                    }
                }
                if (ok && any && p0g >= W - 1) {
                    bool fine = true;
#pragma unroll
                    for (int m = 1; m < W; ++m) {
                        int64_t lb, off;
                        split_n(a, p0g - m, p0g - m < (1ll << 31), lb, off);
                        if (lb >= a.max_blocks) {
                            fine = false;
                        } else {
                            const int32_t b = __ldg(a.bt + static_cast<int64_t>(reqg) * a.bt_rs + lb);
                            fine = fine && b >= 0 && b < a.num_blocks;
                        }
                    }
                    staged = fine;
                    split = q0g - (t0 + i0) > 0 ? q0g - (t0 + i0) : 0;
                }
            }
#pragma unroll
            for (int uu = 0; uu < kTokPerWarp; ++uu) {
                if (staged && uu >= split) continue;  // taken below
                const int code_u = __shfl_sync(0xffffffffu, code, uu);
                const int64_t ins_u = __shfl_sync(0xffffffffu, ins, uu);
                if (code_u == kSkip) continue;  // PAD row or past T
                const int i = i0 + uu;
                const int t = t0 + i;
                float acc[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
                if (code_u == kFast) {
#pragma unroll
                    for (int d = W - 1; d >= 0; --d) wr.fma(acc, d, rows[uu + W - 1 - d]);
                } else if constexpr (TAPS) {
                    // Each tap from its table entry: an x row of the tile, a
                    // cache slot, or zero; the entries come from shared
                    // memory, so every cache tap is one dependent trip.
                    const int64_t *row = mtab + i * (W - 1);
                    const unsigned bad = tab_flags<W>(row, t, mslot[i], slots_total);
                    if (bad) {
                        if (a.err && active) atomicOr(a.err, static_cast<int>(bad));
                        continue;
                    }
#pragma unroll
                    for (int d = W - 1; d >= 1; --d) {
                        const int64_t e = row[d - 1];
                        if (e == SCONV_TAP_X) {
                            wr.fma(acc, d, rows[uu + W - 1 - d]);
                        } else if (e >= 0) {
                            int64_t blk, off;
                            split_n(a, e, a.slots32 != 0, blk, off);
                            P ct;
                            ct.load_nc(cache + blk * a.cs0 + off * a.cs2 + lane);
                            wr.fma(acc, d, ct);
                        }
                    }
                    wr.fma(acc, 0, rows[uu + W - 1]);
                } else {
                    // Taps before the request's first row come from the cache
                    // (zero before position 0), or an index is out of range.
                    const int64_t slot = mslot[i];
                    const int64_t pos = mpos[i];
                    const int req = msid[i];
                    const int q0 = mqs[i];
                    unsigned bad = 0;
                    if (slot < 0 || slot >= slots_total) bad |= SCONV_EFLAG_SLOT;
                    if (req < 0 || req >= a.num_reqs) bad |= SCONV_EFLAG_REQUEST;
                    if (q0 < 0 || q0 > t) bad |= SCONV_EFLAG_QUERY_START;
                    if (pos < 0) bad |= SCONV_EFLAG_POSITION;
                    // Each cache tap is accumulated as it arrives; a bad
                    // block-table index adds its flag (the union over all
                    // taps, as the token kernel reports) and skips the token.
                    if (!bad) {
#pragma unroll
                        for (int d = W - 1; d >= 0; --d) {
                            if (d == 0 || t - d >= q0) {
                                wr.fma(acc, d, rows[uu + W - 1 - d]);
                            } else if (pos - d >= 0) {
                                P ct;
                                const unsigned e = load_cache_tap<E, VEC>(a, req, pos - d, lane, ct);
                                bad |= e;
                                if (!e) wr.fma(acc, d, ct);
                            }
                        }
                    }
                    if (bad) {
                        if (a.err && active) atomicOr(a.err, static_cast<int>(bad));
                        continue;
                    }
                }
                float xc[VEC];
                rows[uu + W - 1].to_float(xc);
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    float y = acc[v];
                    if (SILU) y = silu<E>(y);
                    if (RESID) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
                    acc[v] = y;
                }
                P o;
                o.from_float(acc);
                if (active) {
                    o.store(out + static_cast<int64_t>(t) * a.out_rs + c);
                    rows[uu + W - 1].store(cache + ins_u + lane);
                }
            }
            if (staged) {
                // Window row k holds x row t0 - (W-1) + i0 + k; the rows
                // q0g - m (m = 1..W-1) become the cache rows of positions
                // p0g - m (their block-table entries checked above).
                const int ur = q0g - (t0 + i0);
#pragma unroll
                for (int k = 0; k < kTokPerWarp + W - 1; ++k) {
                    const int m = ur + W - 1 - k;
                    if (k >= split && m >= 1 && m <= W - 1) {
                        int64_t lb, off;
                        split_n(a, p0g - m, p0g - m < (1ll << 31), lb, off);
                        const int32_t b = __ldg(a.bt + static_cast<int64_t>(reqg) * a.bt_rs + lb);
                        rows[k].load_nc(cache + static_cast<int64_t>(b) * a.cs0 + off * a.cs2 + lane);
                    }
                }
#pragma unroll
                for (int uu = 0; uu < kTokPerWarp; ++uu) {
                    if (uu < split) continue;
                    const int code_u = __shfl_sync(0xffffffffu, code, uu);
                    const int64_t ins_u = __shfl_sync(0xffffffffu, ins, uu);
                    if (code_u == kSkip) continue;
                    float acc[VEC];
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
#pragma unroll
                    for (int d = W - 1; d >= 0; --d) wr.fma(acc, d, rows[uu + W - 1 - d]);
                    float xc[VEC];
                    rows[uu + W - 1].to_float(xc);
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        float y = acc[v];
                        if (SILU) y = silu<E>(y);
                        if (RESID) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
                        acc[v] = y;
                    }
                    P o;
                    o.from_float(acc);
                    if (active) {
                        o.store(out + static_cast<int64_t>(t0 + i0 + uu) * a.out_rs + c);
                        rows[uu + W - 1].store(cache + ins_u + lane);
                    }
                }
            }
        }
        // This warp is done with stage s.  The producer refills the stage
        // of the previous tile once all eight warps have released it, so a
        // warp never waits for the others to finish the tile it is on.
        __syncwarp();
        if (lane_id == 0) mbar_arrive(&empty[s]);
        next = k + 1;
        if (threadIdx.x == 0 && k >= 1 && k - 1 + STAGES < my) {
            const int j = k - 1;
            if (mbar_wait(&empty[j % STAGES], (j / STAGES) & 1)) {
                issue(j + STAGES);
            } else {
                if (a.err) atomicOr(a.err, static_cast<int>(SCONV_EFLAG_TIMEOUT));
                alive = false;
                break;
            }
        }
    }
    if (!alive && threadIdx.x == 0) {
        // Let the copies this block issued and has not consumed land before
        // its shared memory is released (each wait bounded).
        for (int j = next; j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
    }
}

bool encode_1d(CUtensorMap *m, CUtensorMapDataType type, const void *base, int64_t n,
               unsigned box_elems = kBT) {
    const cuuint64_t dim[1] = {static_cast<cuuint64_t>(n)};
    const cuuint32_t box[1] = {box_elems};
    const cuuint32_t elem[1] = {1};
    const cuuint64_t no_strides[1] = {0};  // rank 1 has no strides, but the array must exist
    return encode_fn()(m, type, 1, const_cast<void *>(base), dim, no_strides, box, elem,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kLaunchStages = 4;

int gcd_int(int64_t x, int64_t y) {
    while (y != 0) {
        const int64_t r = x % y;
        x = y;
        y = r;
    }
    return static_cast<int>(x);
}

template <typename E, int W, bool SILU, bool RESID, bool TAPS>
cudaError_t launch_flags(const FusedArgs &a, const TmaMaps &maps, cudaStream_t stream) {
    constexpr int S = kLaunchStages;
    constexpr int smem =
        kStages_smem<W, S, TAPS>() + (kCachesWeights<E, W> ? kWeightCacheBytes : 0);
    auto kernel = fused_tma_kernel<E, W, S, SILU, RESID, TAPS>;
    // Resident blocks per SM and the SM count, once per process and kernel
    // (the grid is a function of the device and of T and C only).
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    static int per_sm = 1, sms = 148;
    std::call_once(once, [&] {
        attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (attr != cudaSuccess) return;
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) !=
                cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    });
    if (attr != cudaSuccess) return attr;
    // One block per resident slot, at most one per unit.
    const int64_t ntiles = (a.T + kBT - 1) / kBT;
    const int64_t ncb = (a.C + kBC<E> - 1) / kBC<E>;
    int64_t grid = static_cast<int64_t>(sms) * per_sm;
    if (grid > ntiles * ncb) grid = ntiles * ncb;
    // A block visits ncb / gcd(grid, ncb) channel blocks in turn.
    const int period = static_cast<int>(ncb / gcd_int(grid, ncb));
    const int ncache = (kCachesWeights<E, W> && period > 1 &&
                        period * W * 512 <= kWeightCacheBytes)
                           ? period
                           : 0;
    return launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                      static_cast<size_t>(kStages_smem<W, S, TAPS>() + ncache * W * 512),
                      stream, a, maps, ncache);
}

template <typename E, int W, bool TAPS>
cudaError_t launch_w(const FusedArgs &a, const TmaMaps &maps, cudaStream_t stream) {
    if (a.silu) {
        return a.resid ? launch_flags<E, W, true, true, TAPS>(a, maps, stream)
                       : launch_flags<E, W, true, false, TAPS>(a, maps, stream);
    }
    return a.resid ? launch_flags<E, W, false, true, TAPS>(a, maps, stream)
                   : launch_flags<E, W, false, false, TAPS>(a, maps, stream);
}

// TAPS: the resolved-tap form (a.taps, a.slot; no positions, block table,
// seq_idx or query_start).
template <typename E, bool TAPS>
cudaError_t launch_typed(const FusedArgs &a, cudaStream_t stream, bool &used) {
    constexpr int e = static_cast<int>(sizeof(E));
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (a.W < 1 || a.W > 8 || a.C < kBC<E> || encode_fn() == nullptr) return cudaSuccess;
    if (!al16(a.x) || (a.x_rs * e) % 16 != 0 || !al16(a.slot)) return cudaSuccess;
    if (TAPS ? !al16(a.taps)
             : (!al16(a.positions) || !al16(a.seq_idx) || !al16(a.qstart)))
        return cudaSuccess;
    // The table's tile coordinate t0 * (W-1) is a 32-bit copy coordinate.
    if (TAPS && static_cast<int64_t>(a.T) * (a.W - 1) >= (1ll << 31)) return cudaSuccess;
    TmaMaps maps;
    {
        const cuuint64_t dim[2] = {static_cast<cuuint64_t>(a.C), static_cast<cuuint64_t>(a.T)};
        const cuuint64_t stride[1] = {static_cast<cuuint64_t>(a.x_rs) * e};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBC<E>),
                                   static_cast<cuuint32_t>(kBT + a.W - 1)};
        const cuuint32_t elem[2] = {1, 1};
        const CUtensorMapDataType type =
            e == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        if (encode_fn()(&maps.x, type, 2, const_cast<void *>(a.x), dim, stride, box, elem,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaSuccess;
    }
    if (TAPS) {
        if (!encode_1d(&maps.slot, CU_TENSOR_MAP_DATA_TYPE_INT64, a.slot, a.T) ||
            (a.W > 1 && !encode_1d(&maps.tab, CU_TENSOR_MAP_DATA_TYPE_INT64, a.taps,
                                   static_cast<int64_t>(a.T) * (a.W - 1),
                                   static_cast<unsigned>(kBT * (a.W - 1)))))
            return cudaSuccess;
    } else if (!encode_1d(&maps.pos, CU_TENSOR_MAP_DATA_TYPE_INT64, a.positions, a.T) ||
               !encode_1d(&maps.slot, CU_TENSOR_MAP_DATA_TYPE_INT64, a.slot, a.T) ||
               !encode_1d(&maps.sid, CU_TENSOR_MAP_DATA_TYPE_INT32, a.seq_idx, a.T) ||
               !encode_1d(&maps.qs, CU_TENSOR_MAP_DATA_TYPE_INT32, a.qstart, a.T)) {
        return cudaSuccess;
    }
    used = true;
    switch (a.W) {
        case 1: return launch_w<E, 1, TAPS>(a, maps, stream);
        case 2: return launch_w<E, 2, TAPS>(a, maps, stream);
        case 3: return launch_w<E, 3, TAPS>(a, maps, stream);
        case 4: return launch_w<E, 4, TAPS>(a, maps, stream);
        case 5: return launch_w<E, 5, TAPS>(a, maps, stream);
        case 6: return launch_w<E, 6, TAPS>(a, maps, stream);
        case 7: return launch_w<E, 7, TAPS>(a, maps, stream);
        default: return launch_w<E, 8, TAPS>(a, maps, stream);
    }
}

}  // namespace

cudaError_t launch_fused_tma(const FusedArgs &a, bool bf16_data, cudaStream_t stream,
                             bool &used) {
    used = false;
    return bf16_data ? launch_typed<bf16, false>(a, stream, used)
                     : launch_typed<float, false>(a, stream, used);
}

cudaError_t launch_fused_tma_taps(const FusedArgs &a, bool bf16_data, cudaStream_t stream,
                                  bool &used) {
    used = false;
    return bf16_data ? launch_typed<bf16, true>(a, stream, used)
                     : launch_typed<float, true>(a, stream, used);
}

}  // namespace sconv
