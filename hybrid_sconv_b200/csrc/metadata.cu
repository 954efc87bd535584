// metadata.cu -- per-token request index and request start in one launch
// ("vllm.models.inkling.nvidia.ops.sconv", sconv_seq_metadata), sm_100a.
//
// One thread per token row.  The request is the last r < num_reqs with
// query_start_loc[r] <= t, found by binary search; when the offsets table
// is small each block first stages it in shared memory so the search's
// dependent loads hit shared memory instead of L2.  A second entry point
// runs the same lookup ahead of its wait on the stream.  A third kernel
// also resolves every token's pre-forward taps into a table.
#include "common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

constexpr int kThreads = 256;
constexpr int kSmemReqs = 4096;  // stage query_start_loc when num_reqs <= this

// AHEAD = false waits for the kernels before it on the stream, then works.
// AHEAD = true works first and waits at its end: its completion, which the
// next kernel waits for, still follows theirs, while the lookup overlaps
// them.  It is valid only when none of the kernels that may still be running
// writes query_start_loc or touches the two outputs (one metadata buffer set
// per step in flight).
template <bool AHEAD>
__global__ void __launch_bounds__(kThreads)
seq_metadata_kernel(const int32_t *__restrict__ qsl, int num_reqs, int num_actual,
                    int num_padded, int32_t *__restrict__ seq_idx,
                    int32_t *__restrict__ query_start, int staged) {
    extern __shared__ int32_t s_qsl[];
    // Let the next kernel (typically the fused step that reads these
    // buffers) launch at once: its own wait still orders it after this
    // kernel, and it gets this kernel's whole wait to prefetch.  Then pull
    // the offsets table into L2 while the preceding kernel drains.
    pdl_trigger();
    if (!AHEAD) {
        for (int i = threadIdx.x * 32; i < num_reqs; i += blockDim.x * 32) prefetch_l2(qsl + i);
        pdl_wait();
    }
    if (staged) {
        for (int i = threadIdx.x; i < num_reqs; i += blockDim.x) s_qsl[i] = __ldg(qsl + i);
        __syncthreads();
    }
    const int32_t *q = staged ? s_qsl : qsl;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < num_padded) {
        if (t >= num_actual) {
            seq_idx[t] = 0;
            query_start[t] = 0;
        } else {
            // Invariant: the answer lies in [lo, hi]; q[lo] <= t is assumed for lo = 0.
            int lo = 0, hi = num_reqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (q[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            seq_idx[t] = lo;
            query_start[t] = q[lo];
        }
    }
    if (AHEAD) pdl_wait();  // every thread: the grid completes after its predecessor
}

// Tap resolution, one thread per token row ("vllm.models.inkling.nvidia.ops.sconv",
// module docstring: a tap in the current forward comes from x, an earlier
// one from the cache through block_table[req, src / N] at offset src % N, a
// tap before position 0 is zero).  The request and its first row come from
// the same binary search as above, or are the token itself in the decode
// form.  Row t of the table holds, for lag d = 1..W-1, SCONV_TAP_X,
// SCONV_TAP_ZERO, the flat cache slot b*N + src % N, or -(bits << 8) at every
// lag when the token cannot be resolved.  A thread issues its W-1
// block-table loads together, so the lookup is two dependent accesses
// (positions and query_start_loc, then the block table).
template <bool AHEAD, bool DECODE, int MAXW>
__global__ void __launch_bounds__(kThreads) seq_metadata_taps_kernel(const TapResolveArgs a) {
    extern __shared__ int32_t s_qsl[];
    pdl_trigger();  // as in seq_metadata_kernel
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const bool live = t < a.num_actual;
    if (!AHEAD) {
        if (!DECODE)
            for (int i = threadIdx.x * 32; i < a.num_reqs; i += blockDim.x * 32)
                prefetch_l2(a.qsl + i);
        if (live && (threadIdx.x & 15) == 0) {
            prefetch_l2(a.positions + t);
            prefetch_l2(a.slot + t);
        }
        pdl_wait();
    }
    int64_t pos = 0, slot = -1;
    if (live) {
        pos = __ldg(a.positions + t);
        slot = __ldg(a.slot + t);
    }
    if (!DECODE && a.staged) {
        for (int i = threadIdx.x; i < a.num_reqs; i += blockDim.x) s_qsl[i] = __ldg(a.qsl + i);
        __syncthreads();
    }
    if (t < a.num_padded) {
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
    if (AHEAD) pdl_wait();  // every thread: the grid completes after its predecessor
}

template <bool AHEAD, bool DECODE>
cudaError_t launch_taps_w(const TapResolveArgs &a, size_t smem, cudaStream_t stream) {
    const int blocks = (a.num_padded + kThreads - 1) / kThreads;
    if (a.W <= 4)
        return launch_pdl(seq_metadata_taps_kernel<AHEAD, DECODE, 4>, dim3(blocks),
                          dim3(kThreads), smem, stream, a);
    return launch_pdl(seq_metadata_taps_kernel<AHEAD, DECODE, 8>, dim3(blocks), dim3(kThreads),
                      smem, stream, a);
}

}  // namespace

cudaError_t launch_seq_metadata_taps(TapResolveArgs &a, bool ahead, cudaStream_t stream) {
    a.divN = FastDiv::make(static_cast<uint32_t>(a.N));
    const bool decode = a.qsl == nullptr;
    a.staged = !decode && a.num_reqs <= kSmemReqs ? 1 : 0;
    const size_t smem = a.staged ? static_cast<size_t>(a.num_reqs) * sizeof(int32_t) : 0;
    if (ahead)
        return decode ? launch_taps_w<true, true>(a, smem, stream)
                      : launch_taps_w<true, false>(a, smem, stream);
    return decode ? launch_taps_w<false, true>(a, smem, stream)
                  : launch_taps_w<false, false>(a, smem, stream);
}

cudaError_t launch_seq_metadata(const int32_t *qsl, int num_reqs, int num_actual, int num_padded,
                                int32_t *seq_idx, int32_t *query_start, bool ahead,
                                cudaStream_t stream) {
    // With no actual tokens the search never runs; one entry keeps the
    // staging loop and the search bounds well defined.
    const int nr = num_reqs > 0 ? num_reqs : 1;
    const int staged = nr <= kSmemReqs ? 1 : 0;
    const size_t smem = staged ? static_cast<size_t>(nr) * sizeof(int32_t) : 0;
    const int blocks = (num_padded + kThreads - 1) / kThreads;
    if (ahead)
        return launch_pdl(seq_metadata_kernel<true>, dim3(blocks), dim3(kThreads), smem, stream,
                          qsl, nr, num_actual, num_padded, seq_idx, query_start, staged);
    return launch_pdl(seq_metadata_kernel<false>, dim3(blocks), dim3(kThreads), smem, stream, qsl,
                      nr, num_actual, num_padded, seq_idx, query_start, staged);
}

}  // namespace sconv
