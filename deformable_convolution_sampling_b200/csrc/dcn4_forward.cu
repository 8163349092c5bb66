// dcn4_forward.cu — forward kernel of the DCNv4 core spatial aggregation.
//
// y_g(p0) = sum_k m_gk * bilinear(x_g, p0 + p_k + s*dp_gk)  (CSDN summary of
// "Efficient Deformable ConvNets", section 1.2 equation without the softmax of
// section 2.1).
//
// Mapping.  A CTA owns a TH x TW tile of output pixels of one image (all
// groups), so the samples of its threads fall in a compact window of the input
// that stays in L1.  The tile's offset_mask rows are copied to shared memory
// once with 16-byte streaming loads (not kept in L1), so each
// (pixel, group, k) triple is read from HBM exactly once.  One thread handles
// one (pixel, group, slice), a slice being the VEC x 16 bytes of channels the
// thread owns (nslice slices cover the group's C' channels).  For each of the
// K points the thread forms the location, the bilinear cell and four
// mask-folded weights once, then gathers the four corner slices with one
// 256-bit load each (a whole 32-byte sector per thread; the groups of a pixel
// are adjacent lanes, so a warp's loads spread over distinct slots of the L1
// lines) and accumulates in fp32 with packed f32x2 FMAs: the coefficient reuse
// and vector loads of section 2.2 ("消除冗余工作量", "消除冗余内存指令").
// Nothing is written but the output, with 256-bit stores.
#include "dcn4_common.cuh"

namespace dcn4 {
namespace {

// acc += wt * (the VEC x 16 bytes of channels at src).  VEC == 2 reads the
// whole 32-byte slice with one 256-bit load.
template <typename T, int VEC>
__device__ __forceinline__ void accumulate(float2* acc, const T* src, float wt) {
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

// KH, KW > 0: compile-time grid size (fully unrolled) and RC = remove_center;
// KH = KW = 0: sizes and remove_center from g.
template <typename T, int VEC, int KH, int KW, bool RC>
#ifndef DCN4_FWD_MIN_BLOCKS
#define DCN4_FWD_MIN_BLOCKS 3
#endif
__global__ void __launch_bounds__(256, DCN4_FWD_MIN_BLOCKS) forward_kernel(const Geometry g, const T* __restrict__ value,
                                                      const T* __restrict__ om, T* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    T* om_s = reinterpret_cast<T*>(smem);

    const Tile t = tile_of_block(g);
    stage_tile_rows(om_s, om, g, t);
    __syncthreads();

    // Thread -> (pixel of the tile, group, slice); the groups of one pixel are
    // adjacent lanes, so their corner slices sit at distinct offsets of a line.
    const int lanes_pp = g.G * g.nslice;
    const int lp = threadIdx.x / lanes_pp;
    const int py = lp / g.TW;
    const int px = lp - py * g.TW;
    if (py >= t.th || px >= t.tw) return;
    const int r = threadIdx.x - lp * lanes_pp;
    const int grp = r / g.nslice;
    const int sl = r - grp * g.nslice;
    const int ho = t.ho0 + py, wo = t.wo0 + px;

    const int K = KH > 0 ? KH * KW - (RC ? 1 : 0) : g.K;
    const int kh = KH > 0 ? KH : g.kh;
    const int kw = KW > 0 ? KW : g.kw;
    const bool rc = KH > 0 ? RC : g.remove_center != 0;
    const T* row = om_s + lp * g.P + grp * 3 * K;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* img = value + static_cast<long long>(t.n) * g.H * g.W * g.C + ch_off;
    const int hb = ho * g.sh - g.ph, wb = wo * g.sw - g.pw;

    float2 acc[PAIRS];
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) acc[i] = make_float2(0.f, 0.f);

    int k = 0;
#pragma unroll
    for (int iw = 0; iw < kw; ++iw) {
        const float wbase = static_cast<float>(wb + iw * g.dw);
#pragma unroll
        for (int ih = 0; ih < kh; ++ih) {
            if (rc && iw == kw / 2 && ih == kh / 2) continue;
            const float dx = to_f32(row[2 * k]);
            const float dy = to_f32(row[2 * k + 1]);
            const float m = to_f32(row[2 * K + k]);
            ++k;
            const float h = __fmaf_rn(g.s, dy, static_cast<float>(hb + ih * g.dh));
            const float w = __fmaf_rn(g.s, dx, wbase);
            const Cell<T> cell = bilinear_cell(g, img, h, w);
            const float b = m * cell.lh, a = m - b;  // m (1 - lh), m lh
            const float wl = 1.f - cell.lw;
            accumulate<T, VEC>(acc, cell.c[0], a * wl);
            accumulate<T, VEC>(acc, cell.c[1], a * cell.lw);
            accumulate<T, VEC>(acc, cell.c[2], b * wl);
            accumulate<T, VEC>(acc, cell.c[3], b * cell.lw);
        }
    }

    T* dst = out + ((static_cast<long long>(t.n) * g.Ho + ho) * g.Wo + wo) * g.C + ch_off;
    if constexpr (VEC == 2) {
        st_global32(dst, pack(acc, T()), pack(acc + EPV / 2, T()));
    } else {
        st_global(dst, pack(acc, T()));
    }
}

template <typename T, int VEC, int KH, int KW, bool RC>
cudaError_t launch_typed(const Geometry& g, const void* value, const void* om, void* out, cudaStream_t stream) {
    const size_t smem = forward_smem_bytes(g, sizeof(T));
    auto kern = forward_kernel<T, VEC, KH, KW, RC>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const long long blocks = static_cast<long long>(g.N) * g.tiles_h * g.tiles_w;
    const int threads = (g.pix_per_cta * g.G * g.nslice + 31) / 32 * 32;
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(g, static_cast<const T*>(value),
                                                                   static_cast<const T*>(om), static_cast<T*>(out));
    return cudaGetLastError();
}

template <typename T, int VEC>
cudaError_t launch_grid(const Geometry& g, const void* value, const void* om, void* out, cudaStream_t stream) {
    if (g.kh == 3 && g.kw == 3) {
        return g.remove_center ? launch_typed<T, VEC, 3, 3, true>(g, value, om, out, stream)
                               : launch_typed<T, VEC, 3, 3, false>(g, value, om, out, stream);
    }
    return launch_typed<T, VEC, 0, 0, false>(g, value, om, out, stream);
}

template <typename T>
cudaError_t launch_vec(const Geometry& g, int vec, const void* value, const void* om, void* out, cudaStream_t stream) {
    return vec == 2 ? launch_grid<T, 2>(g, value, om, out, stream) : launch_grid<T, 1>(g, value, om, out, stream);
}

}  // namespace

size_t forward_smem_bytes(const Geometry& g, int elem_bytes) {
    return static_cast<size_t>(g.pix_per_cta) * g.P * elem_bytes;
}

cudaError_t launch_forward(const Geometry& g, int dtype, const void* value, const void* om, void* out,
                           cudaStream_t stream) {
    const int vec = g.vec;
    switch (dtype) {
        case 0: return launch_vec<float>(g, vec, value, om, out, stream);
        case 1: return launch_vec<__half>(g, vec, value, om, out, stream);
        case 2: return launch_vec<__nv_bfloat16>(g, vec, value, om, out, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
