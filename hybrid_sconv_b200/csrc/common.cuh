// common.cuh -- shared device helpers of the sconv library (sm_100a).
//
// Data moves in "packs": VEC consecutive channel elements of one row that
// travel as a single 16-byte transaction (8 bf16 or 4 fp32), or as one
// element when a layout is not 16-byte aligned.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sconv {

using bf16 = __nv_bfloat16;

template <typename E>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte pack
};
template <>
struct Elem<bf16> {
    static constexpr int kVec = 8;
};

// VEC elements of type E held in registers as raw bits.
template <typename E, int VEC>
struct Pack;

// 16-byte pack: four 32-bit words.
template <typename E>
struct Pack16 {
    uint4 u;
    __device__ __forceinline__ void load_nc(const E *p) {
        u = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void store(E *p) const {
        *reinterpret_cast<uint4 *>(p) = u;
    }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
};

template <>
struct Pack<bf16, 8> : Pack16<bf16> {
    // bf16 is the upper half of an fp32, so the widening is exact.
    __device__ __forceinline__ void to_float(float (&f)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ void from_float(const float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        u = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct Pack<float, 4> : Pack16<float> {
    __device__ __forceinline__ void to_float(float (&f)[4]) const {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ void from_float(const float (&f)[4]) {
        u = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                       __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

// One-element packs for layouts that are not 16-byte aligned.
template <>
struct Pack<float, 1> {
    float v;
    __device__ __forceinline__ void load_nc(const float *p) { v = __ldg(p); }
    __device__ __forceinline__ void store(float *p) const { *p = v; }
    __device__ __forceinline__ void zero() { v = 0.f; }
    __device__ __forceinline__ void to_float(float (&f)[1]) const { f[0] = v; }
    __device__ __forceinline__ void from_float(const float (&f)[1]) { v = f[0]; }
};

template <>
struct Pack<bf16, 1> {
    unsigned short v;
    __device__ __forceinline__ void load_nc(const bf16 *p) {
        v = __ldg(reinterpret_cast<const unsigned short *>(p));
    }
    __device__ __forceinline__ void store(bf16 *p) const {
        *reinterpret_cast<unsigned short *>(p) = v;
    }
    __device__ __forceinline__ void zero() { v = 0; }
    __device__ __forceinline__ void to_float(float (&f)[1]) const {
        f[0] = __uint_as_float(static_cast<uint32_t>(v) << 16);
    }
    __device__ __forceinline__ void from_float(const float (&f)[1]) {
        bf16 h = __float2bfloat16_rn(f[0]);
        v = *reinterpret_cast<unsigned short *>(&h);
    }
};

__device__ __forceinline__ float load_weight(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load_weight(const bf16 *p) {
    return __uint_as_float(
        static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short *>(p))) << 16);
}

// Unsigned 32-bit division by a divisor fixed for the whole launch, with one
// multiply-high, a subtract, an add and two shifts: the round-up method of
// Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication" (PLDI 1994), exact for every 32-bit dividend.  For d > 1,
// with l = ceil(log2 d): m = floor(2^32 * (2^l - d) / d) + 1 and
// q = (t + ((n - t) >> 1)) >> (l - 1), t = mulhi(m, n).  d == 1 uses
// m = 0 and shifts 0, giving q = n.
struct FastDiv {
    uint32_t d, m, s1, s2;
#ifndef __CUDACC_RTC__
    __host__ static FastDiv make(uint32_t d) {
        FastDiv f;
        f.d = d;
        if (d <= 1) {
            f.m = 0;
            f.s1 = 0;
            f.s2 = 0;
            return f;
        }
        uint32_t l = 0;
        while ((1ull << l) < d) ++l;
        f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
        f.s1 = 1;
        f.s2 = l - 1;
        return f;
    }
#endif
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        const uint32_t t = __umulhi(m, n);
        return (t + ((n - t) >> s1)) >> s2;
    }
};

// SiLU of the fp32 convolution, one formula per storage type so that every
// kernel produces the same bits for the same token (the residual that
// follows is added with __fadd_rn, so no kernel contracts it into an FMA).  bf16 outputs: y *
// sigmoid(y) written as h + h * tanh(h) with h = y / 2, one hardware tanh
// (tanh.approx.f32, relative error near 2^-11, far below bf16's 2^-8
// rounding step).  fp32 outputs: y / (1 + e^-y) with CUDA's fast exp and
// divide (about 1e-6 relative).
template <typename E>
__device__ __forceinline__ float silu(float y);
template <>
__device__ __forceinline__ float silu<bf16>(float y) {
    const float h = 0.5f * y;
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(h));
    return fmaf(h, th, h);
}
template <>
__device__ __forceinline__ float silu<float>(float y) {
    return __fdividef(y, 1.f + __expf(-y));
}

// Two independent fp32 FMAs (d_i = a_i * b_i + d_i, each rounded once) in
// one packed sm_100 instruction.
__device__ __forceinline__ void fma2(float &d0, float &d1, float a0, float a1, float b0,
                                     float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Programmatic dependent launch (sm_90+): wait for the grids this one
// depends on to finish and flush their memory, and let the grids that
// depend on this one begin launching.  Both are no-ops when the launch did
// not enable programmatic serialization.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bring a line into L2 without reading it into registers.  Safe before
// pdl_wait(): L2 is the device's point of coherence, so a write by the
// preceding kernel that lands after the prefetch is still what the later
// load sees.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Arguments of one fused launch, validated on the host.  Strides in elements.
struct FusedArgs {
    const void *x;
    int64_t x_rs;
    int T, C;
    const void *w;
    int64_t w_sc, w_sk;
    int W;
    int w_vec;  // 1: weight is [C, W] dense and 16-byte aligned (vector loads)
    void *cache;
    int64_t cs0, cs1, cs2;  // block, head, offset strides (D stride is 1)
    int64_t num_blocks;
    int H, N, D;
    FastDiv divN;     // division by N for 32-bit positions and slots
    int slots32;      // num_blocks * N < 2^31: slots divide in 32 bits
    const int64_t *positions;
    const int32_t *seq_idx;  // unused when every token is its own request
    const int64_t *slot;
    const int32_t *qstart;   // unused when every token is its own request
    const int32_t *bt;
    int64_t bt_rs;
    int num_reqs, max_blocks;
    int off_s, ws;
    int silu, resid;
    void *out;
    int64_t out_rs;
    int32_t *err;
    int strip;        // tokens per thread in the strip kernel
    const int64_t *taps;  // resolved tap table [T, W-1] (sconv_fused_taps only)
};

// The per-step tap resolution (sconv_seq_metadata_taps).
struct TapResolveArgs {
    const int32_t *qsl;       // [num_reqs + 1], or nullptr: token t is request t
    int num_reqs, num_actual, num_padded;
    const int64_t *positions, *slot;
    const int32_t *bt;
    int64_t bt_rs;
    int max_blocks;
    int64_t num_blocks;
    int N, W;
    FastDiv divN;
    int32_t *seq_idx, *qstart;  // either may be nullptr
    int64_t *taps;              // [num_padded, W-1]
    int staged;                 // query_start_loc staged in shared memory
};

struct ExtractArgs {
    const void *src;
    int64_t seq_len;
    int conv_dim;
    int64_t src_ss;
    const int32_t *abs_pos;
    const int32_t *real_count;
    int max_count;
    void *out;
    int64_t out_ss;
    int d_conv;
};

// Conditional SSM state-row gather (scatter_intermediate_ssm).
struct SsmArgs {
    const void *states;
    int64_t num_chunks, state_flat, states_rs;
    const int64_t *idx;
    const int32_t *real_count;
    int max_count;
    void *out;
    int64_t out_rs;
    int32_t *err;
};

// Window extraction from the paged cache.
struct PagedExtractArgs {
    const void *cache;
    int64_t cs0, cs1, cs2, num_blocks;
    int H, N, off_s, ws;
    const int32_t *bt;
    int64_t bt_rs;
    int num_reqs, max_blocks;
    const int32_t *request, *abs_pos, *real_count;
    int max_count;
    void *out;
    int64_t out_ss;
    int d_conv;
    int32_t *err;
};

// Dense-state conv (causal_conv1d_fwd / causal_conv1d_update).  Strides in
// elements; for the update, T is the batch and x_st its row stride.
struct DenseArgs {
    const void *x;
    void *out;
    int64_t x_st, x_sc;
    int T, dim;
    const void *w;
    int64_t w_sc, w_sk;
    int W;
    const void *bias;
    void *st;  // conv state lines, or nullptr
    int64_t s_line, s_c, s_k;
    int L, num_lines;
    const int32_t *qsl;     // [batch+1] (prefill)
    int batch;
    const int32_t *lines;   // [batch] or nullptr (line b)
    const uint8_t *init;    // [batch] or nullptr (prefill)
    const int32_t *seqlens; // [batch] or nullptr (update: circular line)
    int silu;
    int pad;
    int32_t *err;
    // Line layout for 16-byte packs of channels: 0 any (element access),
    // 1 channel-contiguous entries (s_c == 1, one pack per entry),
    // 2 entry-contiguous lines (s_k == 1, s_c == L: a pack's lines are one
    // contiguous run of VEC*L elements).
    int st_mode;
};

// Host-side launchers (return the cudaError_t of the launch).
cudaError_t launch_fused(FusedArgs &a, bool bf16_data, bool vec, bool one_token_per_request,
                         cudaStream_t stream);
// Several streams of one layer (same tokens, metadata and cache; disjoint
// lane ranges) in one launch at decode sizes, else one launch per stream.
cudaError_t launch_fused_streams(FusedArgs *s, int n, bool bf16_data, bool vec,
                                 cudaStream_t stream);
// The TMA-pipelined prefill kernel; sets `used` false (and launches
// nothing) when the call does not meet its layout requirements.
cudaError_t launch_fused_tma(const FusedArgs &a, bool bf16_data, cudaStream_t stream,
                             bool &used);
// The same kernel in the resolved-tap form (a.taps and a.slot in place of
// the paged metadata); `used` as for launch_fused_tma.
cudaError_t launch_fused_tma_taps(const FusedArgs &a, bool bf16_data, cudaStream_t stream,
                                  bool &used);
cudaError_t launch_extract(const ExtractArgs &a, bool bf16_data, bool vec, cudaStream_t stream);
cudaError_t launch_scatter_ssm(const SsmArgs &a, int elem_bytes, bool vec, cudaStream_t stream);
cudaError_t launch_extract_paged(const PagedExtractArgs &a, bool bf16_data, bool vec,
                                 cudaStream_t stream);
// `vec`: x (and out) hold channels at unit stride in 16-byte aligned packs.
cudaError_t launch_dense_fwd(const DenseArgs &a, bool bf16_data, bool vec, cudaStream_t stream);
cudaError_t launch_dense_update(const DenseArgs &a, bool bf16_data, bool vec,
                                cudaStream_t stream);
cudaError_t launch_seq_metadata(const int32_t *qsl, int num_reqs, int num_actual, int num_padded,
                                int32_t *seq_idx, int32_t *query_start, bool ahead,
                                cudaStream_t stream);
cudaError_t launch_seq_metadata_taps(TapResolveArgs &a, bool ahead, cudaStream_t stream);
// Several streams (n >= 1) of one layer with their taps read from a resolved
// table; `ready`: slot_mapping and the table may be read before the wait.
cudaError_t launch_fused_taps(FusedArgs *s, int n, bool bf16_data, bool vec, bool ready,
                              cudaStream_t stream);
// The same (taps read after the wait) with the next step's table built by
// extra blocks of the same launch.
cudaError_t launch_fused_taps_next(FusedArgs *s, int n, bool bf16_data, bool vec,
                                   TapResolveArgs &next, cudaStream_t stream);

// Launch with programmatic stream serialization enabled.
template <typename Kernel, typename... Args>
inline cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace sconv
