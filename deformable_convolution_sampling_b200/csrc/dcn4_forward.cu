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
// Nothing is written but the output, with 256-bit stores.  With softmax the
// masks are logits: before its samples each thread takes the K exponentials of
// its (pixel, group)'s logits once, into its own slots of shared memory (no
// barrier), and the samples read their weights from there.
#include <algorithm>
#include <atomic>

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

// CTAs per SM the forward kernel is compiled for (80 registers a thread).
constexpr int kFwdCtasPerSm = 3;

// SM count of the current device, queried once per device.
cudaError_t sm_count(int* out) {
    static std::atomic<int> cached[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *out = c;
            return cudaSuccess;
        }
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) cached[dev].store(sms, std::memory_order_relaxed);
    *out = sms;
    return cudaSuccess;
}

__device__ __forceinline__ Tile tile_at(const Geometry& g, int idx) {
    const int per_img = g.tiles_h * g.tiles_w;
    Tile t;
    t.n = idx / per_img;
    const int r = idx - t.n * per_img;
    const int ty = r / g.tiles_w;
    const int tx = r - ty * g.tiles_w;
    t.ho0 = ty * g.TH;
    t.wo0 = tx * g.TW;
    t.th = min(g.TH, g.Ho - t.ho0);
    t.tw = min(g.TW, g.Wo - t.wo0);
    return t;
}

// The tile's offset_mask rows into shared memory [TH][TW][P] with cp.async (16 bytes per thread per step).
template <typename T>
__device__ __forceinline__ void stage_tile_async(T* dst_smem, const T* src, const Geometry& g, const Tile& t) {
    const int row_chunks = t.tw * g.P * static_cast<int>(sizeof(T)) / 16;
    const int total = t.th * row_chunks;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int r = i / row_chunks;
        const int c = i - r * row_chunks;
        const long long grow = (static_cast<long long>(t.n) * g.Ho + t.ho0 + r) * g.Wo + t.wo0;
        const char* sp = reinterpret_cast<const char*>(src + grow * g.P) + 16ll * c;
        char* d = reinterpret_cast<char*>(dst_smem + r * g.TW * g.P) + 16 * c;
        const unsigned da = static_cast<unsigned>(__cvta_generic_to_shared(d));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(da), "l"(sp));
    }
    asm volatile("cp.async.commit_group;");
}

// Persistent: a CTA per resident slot loops over the output tiles (tile,
// tile + gridDim.x, ...), copying the next tile's offset_mask rows into the
// other half of a double buffer (cp.async) while it computes the current one.
// KH, KW > 0: compile-time grid size (fully unrolled) and RC = remove_center;
// KH = KW = 0: sizes and remove_center from g.  SM: softmax over the K masks.
template <typename T, int VEC, int KH, int KW, bool RC, bool SM>
__global__ void __launch_bounds__(256, kFwdCtasPerSm) forward_kernel(const Geometry g, const T* __restrict__ value,
                                                      const T* __restrict__ om, T* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    const int tile_elems = g.TH * g.TW * g.P;
    T* bufs[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem) + tile_elems};
    float* e_s = reinterpret_cast<float*>(bufs[1] + tile_elems);  // softmax exponentials [K][threads]
    const int ntiles = g.N * g.tiles_h * g.tiles_w;
    int tile = blockIdx.x;
    if (tile >= ntiles) return;
    stage_tile_async(bufs[0], om, g, tile_at(g, tile));

    const int lanes_pp = g.G * g.nslice;
    const int lp = threadIdx.x / lanes_pp;
    const int py = lp / g.TW;
    const int px = lp - py * g.TW;
    const int r = threadIdx.x - lp * lanes_pp;
    const int grp = r / g.nslice;
    const int sl = r - grp * g.nslice;
    const int K = KH > 0 ? KH * KW - (RC ? 1 : 0) : g.K;
    const int kh = KH > 0 ? KH : g.kh;
    const int kw = KW > 0 ? KW : g.kw;
    const bool rc = KH > 0 ? RC : g.remove_center != 0;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);

    for (int it = 0; tile < ntiles; ++it, tile += gridDim.x) {
        const int next = tile + gridDim.x;
        if (next < ntiles) {
            stage_tile_async(bufs[(it + 1) & 1], om, g, tile_at(g, next));
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const Tile t = tile_at(g, tile);
        const T* om_s = bufs[it & 1];
        if (py < t.th && px < t.tw) {
            const int ho = t.ho0 + py, wo = t.wo0 + px;
            const T* row = om_s + lp * g.P + grp * 3 * K;
            const T* img = value + static_cast<long long>(t.n) * g.H * g.W * g.C + ch_off;
            const int hb = ho * g.sh - g.ph, wb = wo * g.sw - g.pw;
            float2 acc[PAIRS];
#pragma unroll
            for (int i = 0; i < PAIRS; ++i) acc[i] = make_float2(0.f, 0.f);
            float inv = 1.f;
            if constexpr (SM) inv = softmax_exps(row + 2 * K, K, e_s + threadIdx.x, blockDim.x).y;
            int k = 0;
#pragma unroll
            for (int iw = 0; iw < kw; ++iw) {
                const float wbase = static_cast<float>(wb + iw * g.dw);
#pragma unroll
                for (int ih = 0; ih < kh; ++ih) {
                    if (rc && iw == kw / 2 && ih == kh / 2) continue;
                    const float dx = to_f32(row[2 * k]);
                    const float dy = to_f32(row[2 * k + 1]);
                    float m = to_f32(row[2 * K + k]);
                    if constexpr (SM) m = e_s[k * blockDim.x + threadIdx.x] * inv;
                    ++k;
                    const float h = __fmaf_rn(g.s, dy, static_cast<float>(hb + ih * g.dh));
                    const float w = __fmaf_rn(g.s, dx, wbase);
                    const Cell<T> cell = bilinear_cell(g, img, h, w);
                    const float b = m * cell.lh, a = m - b;
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
        __syncthreads();  // the buffer is refilled two tiles later
    }
}

template <typename T, int VEC, int KH, int KW, bool RC, bool SM>
cudaError_t launch_typed(const Geometry& g, const void* value, const void* om, void* out, cudaStream_t stream) {
    const size_t smem = forward_smem_bytes(g, sizeof(T));
    auto kern = forward_kernel<T, VEC, KH, KW, RC, SM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int threads = (g.pix_per_cta * g.G * g.nslice + 31) / 32 * 32;
    int sms = 0;
    e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    // One CTA per resident slot (kFwdCtasPerSm by registers, fewer if the double
    // buffer limits shared memory); each loops over tiles.
    const long long by_smem = static_cast<long long>(227 * 1024) / static_cast<long long>(smem + 1024);
    const long long per_sm = std::max<long long>(1, std::min<long long>(kFwdCtasPerSm, by_smem));
    const long long ntiles = static_cast<long long>(g.N) * g.tiles_h * g.tiles_w;
    const long long blocks = std::min<long long>(ntiles, per_sm * sms);
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(g, static_cast<const T*>(value),
                                                                   static_cast<const T*>(om), static_cast<T*>(out));
    return cudaGetLastError();
}

template <typename T, int VEC, bool SM>
cudaError_t launch_grid(const Geometry& g, const void* value, const void* om, void* out, cudaStream_t stream) {
    if (g.kh == 3 && g.kw == 3) {
        return g.remove_center ? launch_typed<T, VEC, 3, 3, true, SM>(g, value, om, out, stream)
                               : launch_typed<T, VEC, 3, 3, false, SM>(g, value, om, out, stream);
    }
    return launch_typed<T, VEC, 0, 0, false, SM>(g, value, om, out, stream);
}

template <typename T, int VEC>
cudaError_t launch_softmax(const Geometry& g, const void* value, const void* om, void* out, cudaStream_t stream) {
    return g.softmax ? launch_grid<T, VEC, true>(g, value, om, out, stream)
                     : launch_grid<T, VEC, false>(g, value, om, out, stream);
}

template <typename T>
cudaError_t launch_vec(const Geometry& g, int vec, const void* value, const void* om, void* out, cudaStream_t stream) {
    return vec == 2 ? launch_softmax<T, 2>(g, value, om, out, stream) : launch_softmax<T, 1>(g, value, om, out, stream);
}

}  // namespace

size_t forward_smem_bytes(const Geometry& g, int elem_bytes) {
    return 2 * static_cast<size_t>(g.pix_per_cta) * g.P * elem_bytes +                        // double buffer
           (g.softmax ? static_cast<size_t>(g.K) * samples_threads(g) * sizeof(float) : 0);  // exponentials
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
