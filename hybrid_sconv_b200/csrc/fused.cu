// fused.cu -- one-launch cache insert + depthwise causal conv1d over the
// paged sliding-window cache ("vllm.models.inkling.nvidia.ops.sconv",
// module docstring and fused_sconv), for sm_100a.
//
// Work split.  A thread owns one pack (VEC consecutive channels, one 16-byte
// transaction) of TPT consecutive tokens.  A block is CV packs wide and TG
// token groups tall (CV * TG = threads), so the grid is
// (ceil(T / (TG*TPT)), ceil(C / (VEC*CV))): a function of T and C only, which
// keeps every launch capturable in a CUDA graph.
//
// Data movement per thread:
//   * the TPT x rows of its tokens are loaded once, up front, as independent
//     16-byte loads, and kept in a register window; the W-1 rows before the
//     tile (the halo) are loaded only when the tile's first token belongs to
//     a request that began earlier (then every same-forward tap of the tile
//     is a window register, so each x element is read from DRAM once);
//   * taps that precede the token's request in x come from the cache via
//     block_table[request, src / N], or are zero before position 0; they only
//     occur for the first W-1 tokens of each request in this step;
//   * each non-PAD token stores its x pack into its cache slot and its
//     output pack into out -- two 16-byte stores.
// The tap source (x, cache or zero) depends only on the token, so it is
// uniform across the lanes of a warp.  Accumulation is fp32, oldest tap first.
#include "common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

template <typename E, int VEC, int MAXW, int TPT, bool ONE_TOKEN_PER_REQUEST>
__global__ void __launch_bounds__(256)
fused_sconv_kernel(const __grid_constant__ FusedArgs a) {
    using P = Pack<E, VEC>;
    const int nv = a.C / VEC;
    const int pack = blockIdx.y * blockDim.x + threadIdx.x;
    const int tok0 = (blockIdx.x * blockDim.y + threadIdx.y) * TPT;
    if (pack >= nv || tok0 >= a.T) return;

    const E *__restrict__ x = static_cast<const E *>(a.x);
    const E *__restrict__ w = static_cast<const E *>(a.w);
    E *__restrict__ cache = static_cast<E *>(a.cache);
    E *__restrict__ out = static_cast<E *>(a.out);

    const int c = pack * VEC;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    const int W = a.W;

    // ---- per-token metadata (the same address across a warp's lanes) ----
    int64_t pos[TPT], slot[TPT];
    int req[TPT], q0[TPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = tok0 + i;
        if (t < a.T) {
            pos[i] = __ldg(a.positions + t);
            slot[i] = __ldg(a.slot + t);
            if (ONE_TOKEN_PER_REQUEST) {
                req[i] = t;
                q0[i] = t;
            } else {
                req[i] = __ldg(a.seq_idx + t);
                q0[i] = __ldg(a.qstart + t);
            }
        } else {
            pos[i] = 0;
            slot[i] = -1;
            req[i] = 0;
            q0[i] = t;
        }
    }

    // ---- x window: rows tok0-(MAXW-1) .. tok0+TPT-1 ----
    P xs[TPT + MAXW - 1];
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = tok0 + i;
        if (t < a.T) xs[MAXW - 1 + i].load_nc(x + static_cast<int64_t>(t) * a.x_rs + c);
    }
    if (!ONE_TOKEN_PER_REQUEST) {
        // Halo rows are same-forward taps only if the tile's first token's
        // request began before the tile (a later token whose taps reach back
        // past tok0 belongs to that same request).
#pragma unroll
        for (int m = 0; m < MAXW - 1; ++m) {
            const int row = tok0 - (MAXW - 1) + m;
            if (m >= MAXW - W && row >= q0[0] && row >= 0)
                xs[m].load_nc(x + static_cast<int64_t>(row) * a.x_rs + c);
        }
    }

    // ---- weights, indexed by lag d = W-1-k (d = 0 is the current token) ----
    float wr[MAXW][VEC];
#pragma unroll
    for (int d = 0; d < MAXW; ++d) {
#pragma unroll
        for (int v = 0; v < VEC; ++v)
            wr[d][v] = d < W ? load_weight(w + static_cast<int64_t>(c + v) * a.w_sc +
                                           static_cast<int64_t>(W - 1 - d) * a.w_sk)
                             : 0.f;
    }

    const int64_t slots_total = a.num_blocks * a.N;
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = tok0 + i;
        if (t >= a.T) break;
        const int64_t s = slot[i];
        if (s == -1) continue;  // PAD row: no insert, no output

        unsigned bad = 0;
        if (s < 0 || s >= slots_total) bad |= SCONV_EFLAG_SLOT;
        if (!ONE_TOKEN_PER_REQUEST) {
            if (req[i] < 0 || req[i] >= a.num_reqs) bad |= SCONV_EFLAG_REQUEST;
            if (q0[i] < 0 || q0[i] > t) bad |= SCONV_EFLAG_QUERY_START;
        }
        if (pos[i] < 0) bad |= SCONV_EFLAG_POSITION;

        // Pre-forward taps (lag d with row t-d before the request's first row).
        P ct[MAXW];
        if (!bad && t - q0[i] < W - 1) {
            const int32_t *bt_row = a.bt + static_cast<int64_t>(req[i]) * a.bt_rs;
#pragma unroll
            for (int d = 1; d < MAXW; ++d) {
                const int64_t src = pos[i] - d;
                if (d < W && t - d < q0[i] && src >= 0) {
                    const int64_t lb = src / a.N;
                    if (lb >= a.max_blocks) {
                        bad |= SCONV_EFLAG_LOGICAL;
                        continue;
                    }
                    const int32_t b = __ldg(bt_row + lb);
                    if (b < 0 || b >= a.num_blocks) {
                        bad |= SCONV_EFLAG_BLOCK;
                        continue;
                    }
                    ct[d].load_nc(cache + static_cast<int64_t>(b) * a.cs0 +
                                  (src - lb * a.N) * a.cs2 + lane);
                }
            }
        }
        if (bad) {
            if (a.err) atomicOr(a.err, static_cast<int>(bad));
            continue;
        }

        float acc[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
#pragma unroll
        for (int d = MAXW - 1; d >= 0; --d) {
            if (d >= W) continue;
            float f[VEC];
            if (t - d >= q0[i]) {
                xs[MAXW - 1 + i - d].to_float(f);
            } else if (pos[i] - d < 0) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) f[v] = 0.f;
            } else {
                ct[d].to_float(f);
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wr[d][v], f[v], acc[v]);
        }

        float xc[VEC];
        xs[MAXW - 1 + i].to_float(xc);
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            float y = acc[v];
            if (a.silu) y = y / (1.f + expf(-y));
            if (a.resid) y += xc[v];
            acc[v] = y;
        }
        P o;
        o.from_float(acc);
        o.store(out + static_cast<int64_t>(t) * a.out_rs + c);

        const int64_t blk = s / a.N;
        xs[MAXW - 1 + i].store(cache + blk * a.cs0 + (s - blk * a.N) * a.cs2 + lane);
    }
}

// Host-side choice of the tile: threads along channels (CV) and tokens per
// thread (TPT) from T and C only.
struct Tile {
    int cv, tg, tpt;
};

inline int next_pow2(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

Tile choose_tile(int T, int nv, int maxw, bool one_token_per_request) {
    Tile tl;
    tl.cv = next_pow2(nv);
    if (tl.cv < 32) tl.cv = 32;
    if (tl.cv > 256) tl.cv = 256;
    // Many token-packs: give each thread several tokens so halo rows and
    // per-token addressing are amortised; few: one token per thread so the
    // grid still covers every SM.
    const int64_t work = static_cast<int64_t>(T) * nv;
    const int64_t fill = 148LL * 2048;  // threads resident on a full B200
    if (one_token_per_request) {
        tl.tpt = 1;
    } else if (work >= 8 * fill) {
        tl.tpt = maxw <= 4 ? 8 : 4;
    } else if (work >= 4 * fill) {
        tl.tpt = 4;
    } else {
        tl.tpt = 1;
    }
    // Small grids: narrower blocks so more SMs get work.
    int threads = 256;
    const int64_t packs_per_block_row = tl.cv;
    const int64_t blocks_256 =
        ((T + (256 / tl.cv) * tl.tpt - 1) / ((256 / tl.cv) * tl.tpt)) *
        ((nv + packs_per_block_row - 1) / packs_per_block_row);
    if (blocks_256 < 2 * 148 && tl.cv <= 128) threads = 128;
    if (threads < tl.cv) threads = tl.cv;
    tl.tg = threads / tl.cv;
    return tl;
}

template <typename E, int VEC, int MAXW, int TPT, bool ONE>
cudaError_t launch_t(const FusedArgs &a, const Tile &tl, cudaStream_t stream) {
    const int nv = a.C / VEC;
    dim3 block(tl.cv, tl.tg);
    const int64_t tokens_per_block = static_cast<int64_t>(tl.tg) * TPT;
    dim3 grid(static_cast<unsigned>((a.T + tokens_per_block - 1) / tokens_per_block),
              static_cast<unsigned>((nv + tl.cv - 1) / tl.cv));
    fused_sconv_kernel<E, VEC, MAXW, TPT, ONE><<<grid, block, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename E, int VEC, int MAXW>
cudaError_t launch_w(const FusedArgs &a, bool one, cudaStream_t stream) {
    const Tile tl = choose_tile(a.T, a.C / VEC, MAXW, one);
    if (one) return launch_t<E, VEC, MAXW, 1, true>(a, tl, stream);
    switch (tl.tpt) {
        case 8:
            if constexpr (MAXW <= 4) return launch_t<E, VEC, MAXW, 8, false>(a, tl, stream);
            else return launch_t<E, VEC, MAXW, 4, false>(a, tl, stream);
        case 4: return launch_t<E, VEC, MAXW, 4, false>(a, tl, stream);
        default: return launch_t<E, VEC, MAXW, 1, false>(a, tl, stream);
    }
}

template <typename E, int VEC>
cudaError_t launch_v(const FusedArgs &a, bool one, cudaStream_t stream) {
    if (a.W <= 4) return launch_w<E, VEC, 4>(a, one, stream);
    return launch_w<E, VEC, 8>(a, one, stream);
}

}  // namespace

cudaError_t launch_fused(const FusedArgs &a, bool bf16_data, bool vec, bool one,
                         cudaStream_t stream) {
    if (bf16_data) {
        return vec ? launch_v<bf16, 8>(a, one, stream) : launch_v<bf16, 1>(a, one, stream);
    }
    return vec ? launch_v<float, 4>(a, one, stream) : launch_v<float, 1>(a, one, stream);
}

}  // namespace sconv
