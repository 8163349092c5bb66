// dcn4_attn.cu — single-scale deformable attention on sm_100a.
//
// For query q (reference point r_q, pixel coordinates) and group g:
//     y_g(q) = sum_{k<K} A_gk * x_g(r_q + s * dp_gk),
//     A_gk   = softmax over the K points of the logits l_gk
// (CSDN summary of "Efficient Deformable ConvNets", section 1.1: each query
// attends to a selected number of sampling points whose positions and weights
// are dynamic; section 1.2: the DCNv3 weights are a softmax over the points).
// The sampling is the aggregation's: a fp32 fma for the location, the bilinear
// cell of the zero-extended image, 256-bit corner gathers of a group's channels,
// fp32 accumulation (section 2.2 "消除冗余内存指令" notes that the same memory
// optimisations apply to deformable attention).
//
// Forward: a thread per (query, group, 32- or 16-byte channel slice); a CTA
// takes a run of consecutive queries (neighbours in the pixel-centre order of
// an encoder, so their samples share L1 lines) and stages their
// offset_logits rows and reference points in shared memory once.
//
// Backward: the same mapping.  grad of the offsets and logits from the four
// per-corner dot products <gy, v_ab> (reduced over the slices of a group), the
// softmax Jacobian applied to the weight gradients; grad_value scattered with
// vector fp32 reductions into an fp32 accumulator (the workspace for 16-bit
// I/O, grad_value itself for fp32), then rounded once to the I/O dtype.
#include <algorithm>

#include "dcn4_common.cuh"

namespace dcn4 {
namespace {

constexpr int kAttnThreads = 256;

// <gy, the VEC x 16 bytes of channels at src>, in fp32.
template <typename T, int VEC>
__device__ __forceinline__ float attn_dot(const float2* gy, const T* src) {
    constexpr int PAIRS = Elem<T>::per16 / 2;
    uint4 raw[VEC];
    if constexpr (VEC == 2) {
        ld_gather32(src, raw[0], raw[1]);
    } else {
        raw[0] = ld_gather(src);
    }
    float2 d = make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        float2 f[PAIRS];
        unpack(raw[v], f, T());
#pragma unroll
        for (int i = 0; i < PAIRS; ++i) d = __ffma2_rn(gy[v * PAIRS + i], f[i], d);
    }
    return d.x + d.y;
}

template <typename T, int VEC>
__device__ __forceinline__ void attn_accumulate(float2* acc, const T* src, float wt) {
    constexpr int PAIRS = Elem<T>::per16 / 2;
    const float2 w2 = make_float2(wt, wt);
    uint4 raw[VEC];
    if constexpr (VEC == 2) {
        ld_gather32(src, raw[0], raw[1]);
    } else {
        raw[0] = ld_gather(src);
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        float2 f[PAIRS];
        unpack(raw[v], f, T());
#pragma unroll
        for (int i = 0; i < PAIRS; ++i) acc[v * PAIRS + i] = __ffma2_rn(w2, f[i], acc[v * PAIRS + i]);
    }
}

// dst[0..3] += v (fp32, one vector reduction in L2).
__device__ __forceinline__ void red_add4(float* dst, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// The CTA's rows [q0, q0 + nq) of offset_logits (P wide) and their reference
// points into shared memory.
template <typename T>
__device__ __forceinline__ void stage_queries(T* rows, float2* refs, const T* ol, const float* ref, long long q0,
                                              int nq, int P) {
    const int chunks = nq * P * static_cast<int>(sizeof(T)) / 16;
    const char* src = reinterpret_cast<const char*>(ol + q0 * P);
    for (int i = threadIdx.x; i < chunks; i += blockDim.x)
        reinterpret_cast<uint4*>(rows)[i] = ld_stream(src + 16ll * i);
    for (int i = threadIdx.x; i < nq; i += blockDim.x)
        refs[i] = make_float2(ref[2 * (q0 + i)], ref[2 * (q0 + i) + 1]);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kAttnThreads) attn_forward_kernel(const Geometry g, int Nq, int QB,
                                                                    const T* __restrict__ value,
                                                                    const float* __restrict__ ref,
                                                                    const T* __restrict__ ol, T* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    T* rows = reinterpret_cast<T*>(smem);
    float2* refs = reinterpret_cast<float2*>(rows + static_cast<size_t>(QB) * g.P);
    float* e_s = reinterpret_cast<float*>(refs + QB);  // [K][threads]
    const long long total = static_cast<long long>(g.N) * Nq;
    const long long q0 = static_cast<long long>(blockIdx.x) * QB;
    const int nq = static_cast<int>(min(static_cast<long long>(QB), total - q0));
    stage_queries(rows, refs, ol, ref, q0, nq, g.P);
    __syncthreads();
    const int lanes_pq = g.G * g.nslice;
    const int lq = threadIdx.x / lanes_pq;
    if (lq >= nq) return;
    const int r = threadIdx.x - lq * lanes_pq;
    const int grp = r / g.nslice, sl = r - grp * g.nslice;
    const long long qq = q0 + lq;
    const int n = static_cast<int>(qq / Nq);
    const int K = g.K;
    const T* row = rows + static_cast<size_t>(lq) * g.P + grp * 3 * K;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* img = value + static_cast<long long>(n) * g.H * g.W * g.C + ch_off;
    const float2 rp = refs[lq];
    const float inv = softmax_exps(row + 2 * K, K, e_s + threadIdx.x, blockDim.x).y;
    float2 acc[PAIRS];
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) acc[i] = make_float2(0.f, 0.f);
    for (int k = 0; k < K; ++k) {
        const float dx = to_f32(row[2 * k]), dy = to_f32(row[2 * k + 1]);
        const float m = e_s[k * blockDim.x + threadIdx.x] * inv;
        const Cell<T> cell = bilinear_cell(g, img, __fmaf_rn(g.s, dy, rp.y), __fmaf_rn(g.s, dx, rp.x));
        const float b = m * cell.lh, a = m - b;
        const float wl = 1.f - cell.lw;
        attn_accumulate<T, VEC>(acc, cell.c[0], a * wl);
        attn_accumulate<T, VEC>(acc, cell.c[1], a * cell.lw);
        attn_accumulate<T, VEC>(acc, cell.c[2], b * wl);
        attn_accumulate<T, VEC>(acc, cell.c[3], b * cell.lw);
    }
    T* dst = out + qq * g.C + ch_off;
    if constexpr (VEC == 2) {
        st_global32(dst, pack(acc, T()), pack(acc + EPV / 2, T()));
    } else {
        st_global(dst, pack(acc, T()));
    }
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kAttnThreads) attn_backward_kernel(const Geometry g, int Nq, int QB,
                                                                     const T* __restrict__ value,
                                                                     const float* __restrict__ ref,
                                                                     const T* __restrict__ ol,
                                                                     const T* __restrict__ gout, T* __restrict__ gol,
                                                                     float* __restrict__ gacc) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    T* rows = reinterpret_cast<T*>(smem);
    T* grows = rows + static_cast<size_t>(QB) * g.P;  // grad_offset_logits rows of the CTA
    float2* refs = reinterpret_cast<float2*>(grows + static_cast<size_t>(QB) * g.P);
    float* e_s = reinterpret_cast<float*>(refs + QB);  // [K][threads]: exponentials, then <gy, S_k>
    const long long total = static_cast<long long>(g.N) * Nq;
    const long long q0 = static_cast<long long>(blockIdx.x) * QB;
    const int nq = static_cast<int>(min(static_cast<long long>(QB), total - q0));
    stage_queries(rows, refs, ol, ref, q0, nq, g.P);
    for (int i = threadIdx.x; i < nq * g.P; i += blockDim.x) grows[i] = static_cast<T>(0.f);
    __syncthreads();
    const int lanes_pq = g.G * g.nslice;
    const int lq = threadIdx.x / lanes_pq;
    // lanes of a query past the end stay (sampling nothing) so every lane reaches the shuffles
    const bool active = lq < nq;
    const int lqa = active ? lq : 0;
    const int r = threadIdx.x - lq * lanes_pq;
    const int grp = r / g.nslice, sl = r - grp * g.nslice;
    const long long qq = q0 + lqa;
    const int n = static_cast<int>(qq / Nq);
    const int K = g.K;
    const T* row = rows + static_cast<size_t>(lqa) * g.P + grp * 3 * K;
    T* grow = grows + static_cast<size_t>(lqa) * g.P + grp * 3 * K;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* img = value + static_cast<long long>(n) * g.H * g.W * g.C + ch_off;
    float* acc_img = gacc + static_cast<long long>(n) * g.H * g.W * g.C + ch_off;
    const float2 rp = refs[lqa];
    float2 gy[PAIRS];
    {
        const T* src = gout + qq * g.C + ch_off;
        uint4 raw[VEC];
        if constexpr (VEC == 2) {
            ld_gather32(src, raw[0], raw[1]);
        } else {
            raw[0] = ld_gather(src);
        }
#pragma unroll
        for (int v = 0; v < VEC; ++v) unpack(raw[v], gy + v * (EPV / 2), T());
    }
    const float inv = softmax_exps(row + 2 * K, K, e_s + threadIdx.x, blockDim.x).y;
    const bool writer = active && sl == 0;
    float gdot = 0.f;  // sum_k A_k <gy, S_k>
    for (int k = 0; k < K; ++k) {
        const float dx = to_f32(row[2 * k]), dy = to_f32(row[2 * k + 1]);
        const float m = e_s[k * blockDim.x + threadIdx.x] * inv;
        const float h = active ? __fmaf_rn(g.s, dy, rp.y) : -2.f;
        const Cell<T> cell = bilinear_cell(g, img, h, __fmaf_rn(g.s, dx, rp.x));
        float d00 = attn_dot<T, VEC>(gy, cell.c[0]);
        float d01 = attn_dot<T, VEC>(gy, cell.c[1]);
        float d10 = attn_dot<T, VEC>(gy, cell.c[2]);
        float d11 = attn_dot<T, VEC>(gy, cell.c[3]);
        for (int off = g.nslice >> 1; off > 0; off >>= 1) {
            d00 += __shfl_xor_sync(0xffffffffu, d00, off);
            d01 += __shfl_xor_sync(0xffffffffu, d01, off);
            d10 += __shfl_xor_sync(0xffffffffu, d10, off);
            d11 += __shfl_xor_sync(0xffffffffu, d11, off);
        }
        const float hl = 1.f - cell.lh, wl = 1.f - cell.lw;
        const float gw = cell.any ? hl * (wl * d00 + cell.lw * d01) + cell.lh * (wl * d10 + cell.lw * d11) : 0.f;
        // this lane's exponential slot of point k is spent: it keeps <gy, S_k>
        e_s[k * blockDim.x + threadIdx.x] = gw;
        gdot = __fmaf_rn(m, gw, gdot);
        if (!cell.any) continue;
        if (writer) {
            const float sm = g.s * m;
            grow[2 * k] = from_f32<T>(sm * (hl * (d01 - d00) + cell.lh * (d11 - d10)));
            grow[2 * k + 1] = from_f32<T>(sm * (wl * (d10 - d00) + cell.lw * (d11 - d01)));
        }
        // grad_value: m * (corner weight) * gy into each in-image corner
        const float b = m * cell.lh, a = m - b;
        const float wc[4] = {a * wl, a * cell.lw, b * wl, b * cell.lw};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int y = cell.h0 + (c >> 1), x = cell.w0 + (c & 1);
            if (y < 0 || y >= g.H || x < 0 || x >= g.W) continue;
            float* dst = acc_img + (static_cast<long long>(y) * g.W + x) * g.C;
#pragma unroll
            for (int i = 0; i < PAIRS / 2; ++i)
                red_add4(dst + 4 * i, make_float4(wc[c] * gy[2 * i].x, wc[c] * gy[2 * i].y, wc[c] * gy[2 * i + 1].x,
                                                  wc[c] * gy[2 * i + 1].y));
        }
    }
    if (writer) {
        // logit gradients: the softmax Jacobian applied to the weight gradients
        for (int k = 0; k < K; ++k) {
            const float m = softmax_weight(to_f32(row[2 * K + k]), softmax_stats(row + 2 * K, K));
            grow[2 * K + k] = from_f32<T>(m * (e_s[k * blockDim.x + threadIdx.x] - gdot));
        }
    }
    __syncthreads();
    const int chunks = nq * g.P * static_cast<int>(sizeof(T)) / 16;
    char* dst = reinterpret_cast<char*>(gol + q0 * g.P);
    for (int i = threadIdx.x; i < chunks; i += blockDim.x)
        st_global(dst + 16ll * i, reinterpret_cast<const uint4*>(grows)[i]);
}

// grad_value = round(acc), 16 bytes of output per thread.
template <typename T>
__global__ void attn_round_kernel(const float* __restrict__ acc, T* __restrict__ gv, long long n16) {
    constexpr int EPV = Elem<T>::per16;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n16;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        float2 f[EPV / 2];
        const float4* s = reinterpret_cast<const float4*>(acc + i * EPV);
#pragma unroll
        for (int j = 0; j < EPV / 4; ++j) {
            const float4 v = __ldcs(s + j);
            f[2 * j] = make_float2(v.x, v.y);
            f[2 * j + 1] = make_float2(v.z, v.w);
        }
        st_global(gv + i * EPV, pack(f, T()));
    }
}

int attn_queries_per_cta(const Geometry& g) { return std::max(1, kAttnThreads / (g.G * g.nslice)); }

template <typename T, int VEC>
cudaError_t attn_forward_typed(const Geometry& g, int Nq, const void* value, const float* ref, const void* ol,
                               void* out, cudaStream_t stream) {
    const int QB = attn_queries_per_cta(g);
    const size_t smem = attn_smem_bytes(g, sizeof(T), false);
    auto kern = attn_forward_kernel<T, VEC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long blocks = (static_cast<long long>(g.N) * Nq + QB - 1) / QB;
    kern<<<static_cast<unsigned>(blocks), kAttnThreads, smem, stream>>>(g, Nq, QB, static_cast<const T*>(value), ref,
                                                                        static_cast<const T*>(ol), static_cast<T*>(out));
    return cudaGetLastError();
}

template <typename T, int VEC>
cudaError_t attn_backward_typed(const Geometry& g, int Nq, const void* value, const float* ref, const void* ol,
                                const void* gout, void* gvalue, void* gol, float* acc, cudaStream_t stream) {
    const int QB = attn_queries_per_cta(g);
    const size_t smem = attn_smem_bytes(g, sizeof(T), true);
    auto kern = attn_backward_kernel<T, VEC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long blocks = (static_cast<long long>(g.N) * Nq + QB - 1) / QB;
    kern<<<static_cast<unsigned>(blocks), kAttnThreads, smem, stream>>>(
        g, Nq, QB, static_cast<const T*>(value), ref, static_cast<const T*>(ol), static_cast<const T*>(gout),
        static_cast<T*>(gol), acc);
    e = cudaGetLastError();
    if (e != cudaSuccess || sizeof(T) == 4) return e;
    const long long n16 = static_cast<long long>(g.N) * g.H * g.W * g.C / Elem<T>::per16;
    const long long rb = std::min<long long>((n16 + 255) / 256, 148LL * 16);
    attn_round_kernel<T><<<static_cast<unsigned>(std::max<long long>(rb, 1)), 256, 0, stream>>>(acc, static_cast<T*>(gvalue), n16);
    return cudaGetLastError();
}

}  // namespace

size_t attn_smem_bytes(const Geometry& g, int elem_bytes, bool backward) {
    const size_t QB = static_cast<size_t>(attn_queries_per_cta(g));
    return QB * g.P * elem_bytes * (backward ? 2 : 1) + QB * sizeof(float2) +
           static_cast<size_t>(g.K) * kAttnThreads * sizeof(float);
}

cudaError_t launch_attn_forward(const Geometry& g, int dtype, int Nq, const void* value, const float* ref,
                                const void* ol, void* out, cudaStream_t stream) {
    switch (dtype) {
        case 0: return g.vec == 2 ? attn_forward_typed<float, 2>(g, Nq, value, ref, ol, out, stream)
                                  : attn_forward_typed<float, 1>(g, Nq, value, ref, ol, out, stream);
        case 1: return g.vec == 2 ? attn_forward_typed<__half, 2>(g, Nq, value, ref, ol, out, stream)
                                  : attn_forward_typed<__half, 1>(g, Nq, value, ref, ol, out, stream);
        case 2: return g.vec == 2 ? attn_forward_typed<__nv_bfloat16, 2>(g, Nq, value, ref, ol, out, stream)
                                  : attn_forward_typed<__nv_bfloat16, 1>(g, Nq, value, ref, ol, out, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attn_backward(const Geometry& g, int dtype, int Nq, const void* value, const float* ref,
                                 const void* ol, const void* gout, void* gvalue, void* gol, float* acc,
                                 cudaStream_t stream) {
    switch (dtype) {
        case 0: return g.vec == 2 ? attn_backward_typed<float, 2>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream)
                                  : attn_backward_typed<float, 1>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream);
        case 1: return g.vec == 2 ? attn_backward_typed<__half, 2>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream)
                                  : attn_backward_typed<__half, 1>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream);
        case 2: return g.vec == 2
                           ? attn_backward_typed<__nv_bfloat16, 2>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream)
                           : attn_backward_typed<__nv_bfloat16, 1>(g, Nq, value, ref, ol, gout, gvalue, gol, acc, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
