// dcn4_common.cuh — device-side helpers shared by the libdcn4 kernels.
//
// Element access is in 16-byte vectors (8 x fp16/bf16 or 4 x fp32): the C'
// channels of a group are contiguous in the channels-last layout, so one
// 128-bit instruction moves a whole run of them (CSDN summary of "Efficient
// Deformable ConvNets", section 2.2, "消除冗余内存指令").
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace dcn4 {

// Problem geometry with the derived sizes the kernels need (filled on the host).
struct Geometry {
    int N, H, W, G, Cg, C, Ho, Wo, P, K;
    int kh, kw, sh, sw, ph, pw, dh, dw;
    float s;              // offset_scale
    int remove_center;
    int softmax;          // masks are logits normalised by a softmax over the K points
    int vec;              // 16-byte vectors per thread slice: 2 (one 32-byte access) or 1
    int nslice;           // threads cooperating on one (pixel, group): power of two <= 32
    int pix_per_cta;      // output pixels handled by one CTA (= TH * TW)
    long long total_pix;  // N * Ho * Wo
    int TH, TW;           // output tile of one CTA (rows x columns of one image)
    int tiles_h, tiles_w; // tiles per image
    // grad_value pass: input tiles of BH x BW pixels, bthreads threads per CTA,
    // room for bcap sample records in shared memory.
    int BH, BW, btiles_h, btiles_w, bthreads, bcap;
    int brec;  // bytes per sample record: 8 (16-bit dtypes) or 16 (fp32)
    int LW;    // lanes of one strip (one lane per cell column, BW + 1 <= LW): 8, 16 or 32
    int BS;    // pixel rows of one strip segment
    int nseg;  // segments per tile: ceil(BH / BS)
    // Buckets (16-bit dtypes): the grad_offset_mask pass files each sample's
    // record under every grad_value tile whose cells hold it, up to bcap per
    // tile.  bh_magic / bw_magic divide a pixel coordinate by BH / BW with
    // __umulhi (exact for coordinates < 2^24).
    int buckets;
    uint32_t bh_magic, bw_magic;
    // Filing window of the grad_offset_mask CTA: fwin_h tile rows x 2^fwin_wl
    // tile columns (64 tiles).
    int fwin_h, fwin_wl;
    // Forward: offset_mask tiles in flight per CTA (set by the forward's launcher).
    int fbufs;
};

// What the grad_offset_mask pass leaves for the grad_value pass.
//   code        [N, Ho, Wo, G, K]  fp32: the cell code of every sample
// 16-bit dtypes, when g.buckets:
//   tile_count  [N * btiles_h * btiles_w]  records filed per grad_value tile
//               (pre-zeroed; above bcap -- or with kBucketOverflow set -- the
//               tile's bucket is incomplete and the tile rescans the offsets)
//   bucket_pix  [tiles][bcap]  output pixel of the record, (ho << 16) | wo
//   bucket_rec  [tiles][bcap]  bin (group, cell) of the record in the tile |
//               mask bits << 16 | lh << 32 | lw << 48 (16-bit fixed point)
// Arrays a dtype does not use are NULL.
struct SampleArrays {
    uint16_t* code;
    int* tile_count;
    uint32_t* bucket_pix;
    uint64_t* bucket_rec;
    int* diag;  // fallback counters of the grad_value pass (kDiag*)
};
// Counters the grad_value pass keeps per call: tiles whose bucket failed the
// consistency checks (taken by the direct path), tiles that rescanned the
// offsets (bucket overflow, or a sample beyond the filing window), and tiles
// that took the direct path for any reason.
constexpr int kDiagCorruptBucket = 0;
constexpr int kDiagRescan = 1;
constexpr int kDiagDirect = 2;
constexpr int kDiagWords = 4;
constexpr int kBucketOverflow = 1 << 30;

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int per16 = 4;
};
template <>
struct Elem<__half> {
    static constexpr int per16 = 8;
};
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int per16 = 8;
};

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---------------------------------------------------------------------------
// 16-byte vector <-> float pairs
// ---------------------------------------------------------------------------
__device__ __forceinline__ void unpack(const uint4& r, float2* f, float) {
    f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    f[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
}
__device__ __forceinline__ void unpack(const uint4& r, float2* f, __half) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h;
        memcpy(&h, &w[i], 4);
        f[i] = __half22float2(h);
    }
}
__device__ __forceinline__ void unpack(const uint4& r, float2* f, __nv_bfloat16) {
    // bfloat16 is the upper half of a binary32: widen by placing the bits there.
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

__device__ __forceinline__ uint4 pack(const float2* f, float) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
}
__device__ __forceinline__ uint4 pack(const float2* f, __half) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 h = __float22half2_rn(f[i]);
        memcpy(&w[i], &h, 4);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 pack(const float2* f, __nv_bfloat16) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __float22bfloat162_rn(f[i]);
        memcpy(&w[i], &h, 4);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------------------
// Global memory access
// ---------------------------------------------------------------------------

// Read-only gather through L1 (value rows are re-read by neighbouring samples).
__device__ __forceinline__ uint4 ld_gather(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// 32-byte read-only gather (one full sector per thread, sm_100 256-bit load).
__device__ __forceinline__ void ld_gather32(const void* p, uint4& lo, uint4& hi) {
    asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
}

// 32-byte read-only gather that should stay in L1 (evicted last).
__device__ __forceinline__ void ld_keep32(const void* p, uint4& lo, uint4& hi) {
    asm volatile("ld.global.nc.L1::evict_last.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
}
__device__ __forceinline__ uint4 ld_keep16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 2-byte read that bypasses L1 (used once; keeps L1 for the gathers).
__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint64_t ld_stream_u64(const void* p) {
    unsigned long long r;
    asm volatile("ld.global.nc.L1::no_allocate.u64 %0, [%1];" : "=l"(r) : "l"(p));
    return r;
}

// 32-byte store (sm_100 256-bit store).
__device__ __forceinline__ void st_global32(void* p, const uint4& lo, const uint4& hi) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(lo.x), "r"(lo.y),
                 "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
                 : "memory");
}

// Streaming read that is used once (offset_mask rows, grad_out): do not keep in L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_global(void* p, const uint4& v) {
    *reinterpret_cast<uint4*>(p) = v;
}

// Output pixel index -> (n, ho, wo).
__device__ __forceinline__ void pixel_coords(const Geometry& g, long long pix, int& n, int& ho, int& wo) {
    const long long hw = static_cast<long long>(g.Ho) * g.Wo;
    n = static_cast<int>(pix / hw);
    const int rem = static_cast<int>(pix - static_cast<long long>(n) * hw);
    ho = rem / g.Wo;
    wo = rem - ho * g.Wo;
}

// Copies `bytes` (a multiple of 16) of contiguous global memory into shared
// memory with the whole CTA, 16 bytes per thread per step.
__device__ __forceinline__ void stage_rows(void* dst_smem, const void* src, int bytes) {
    uint4* d = reinterpret_cast<uint4*>(dst_smem);
    const char* s = reinterpret_cast<const char*>(src);
    for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) d[i] = ld_stream(s + 16ll * i);
}

// One CTA's output tile: image n, rows [ho0, ho0 + th), columns [wo0, wo0 + tw).
struct Tile {
    int n, ho0, wo0, th, tw;
};

__device__ __forceinline__ Tile tile_of_block(const Geometry& g) {
    const int per_img = g.tiles_h * g.tiles_w;
    Tile t;
    t.n = blockIdx.x / per_img;
    const int r = blockIdx.x - t.n * per_img;
    const int ty = r / g.tiles_w;
    const int tx = r - ty * g.tiles_w;
    t.ho0 = ty * g.TH;
    t.wo0 = tx * g.TW;
    t.th = min(g.TH, g.Ho - t.ho0);
    t.tw = min(g.TW, g.Wo - t.wo0);
    return t;
}

// Copies the P-wide rows of a tile of pixels (row-major [th][tw] in a [*, Ho, Wo, P]
// tensor) into shared memory laid out [TH][TW][P]; 16 bytes per thread per step.
template <typename T>
__device__ __forceinline__ void stage_tile_rows(T* dst_smem, const T* src, const Geometry& g, const Tile& t) {
    const int row_chunks = t.tw * g.P * static_cast<int>(sizeof(T)) / 16;  // 16-byte chunks per tile row
    const int total = t.th * row_chunks;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int r = i / row_chunks;
        const int c = i - r * row_chunks;
        const long long grow = (static_cast<long long>(t.n) * g.Ho + t.ho0 + r) * g.Wo + t.wo0;
        const char* s = reinterpret_cast<const char*>(src + grow * g.P) + 16ll * c;
        char* d = reinterpret_cast<char*>(dst_smem + r * g.TW * g.P) + 16 * c;
        *reinterpret_cast<uint4*>(d) = ld_stream(s);
    }
}

// ---------------------------------------------------------------------------
// Softmax over the K mask logits of one (pixel, group) -- the DCNv3 form of the
// modulation scalars (CSDN summary of "Efficient Deformable ConvNets", section
// 1.2): m_k = exp(l_k - l_max) / sum_j exp(l_j - l_max), in fp32, the sum taken
// in k order.  softmax_stats returns (l_max, 1 / sum) and softmax_weight then
// gives m_k; softmax_exps keeps the K exponentials (e[k * stride]) and returns
// the same (l_max, 1 / sum), m_k being e_k * (1 / sum).  All give the same fp32
// weights.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float2 softmax_stats(const T* logits, int K) {
    float mx = -INFINITY;
    for (int j = 0; j < K; ++j) mx = fmaxf(mx, to_f32(logits[j]));
    float sum = 0.f;
    for (int j = 0; j < K; ++j) sum += expf(to_f32(logits[j]) - mx);
    return make_float2(mx, 1.f / sum);
}
__device__ __forceinline__ float softmax_weight(float logit, float2 stats) {
    return expf(logit - stats.x) * stats.y;
}
template <typename T>
__device__ __forceinline__ float2 softmax_exps(const T* logits, int K, float* e, int stride) {
    float mx = -INFINITY;
    for (int j = 0; j < K; ++j) mx = fmaxf(mx, to_f32(logits[j]));
    float sum = 0.f;
    for (int j = 0; j < K; ++j) {
        const float x = expf(to_f32(logits[j]) - mx);
        e[j * stride] = x;
        sum += x;
    }
    return make_float2(mx, 1.f / sum);
}

// ---------------------------------------------------------------------------
// Bilinear cell of one sample, branch-free
// ---------------------------------------------------------------------------

// 32 zero bytes: the gather address of a corner outside the image, so every
// corner can be loaded unconditionally (its value then contributes 0).  One
// copy per translation unit (device code is not relocatable).
static __device__ __align__(32) const uint4 g_zero_slice[2] = {};

// The four corners of the cell that floor() selects for location (h, w):
// c[0] = (h0, w0), c[1] = (h0, w0+1), c[2] = (h0+1, w0), c[3] = (h0+1, w0+1),
// with bilinear weights wt[] = (1-lh)(1-lw), (1-lh)lw, lh(1-lw), lh lw.  A
// corner outside [0,H) x [0,W) gets the zero slice as its address; a location
// that touches no pixel (h < -1, h >= H, w < -1, w >= W, or NaN) gets it for
// all four.  `img` points at this thread's channels of pixel (0, 0) of the image.
template <typename T>
struct Cell {
    const T* c[4];
    float lh, lw;
    int h0, w0;  // top-left corner of the cell (meaningful when any)
    bool any;    // some corner is inside the image
};

template <typename T>
__device__ __forceinline__ Cell<T> bilinear_cell(const Geometry& g, const T* img, float h, float w) {
    Cell<T> cell;
    cell.any = h >= -1.f && h < static_cast<float>(g.H) && w >= -1.f && w < static_cast<float>(g.W);
    const float hc = cell.any ? h : 0.f, wc = cell.any ? w : 0.f;
    const float h0f = floorf(hc), w0f = floorf(wc);
    cell.lh = hc - h0f;
    cell.lw = wc - w0f;
    const int h0 = static_cast<int>(h0f), w0 = static_cast<int>(w0f);
    cell.h0 = h0;
    cell.w0 = w0;
    const bool y0 = cell.any && h0 >= 0, y1 = cell.any && h0 + 1 < g.H;
    const bool x0 = w0 >= 0, x1 = w0 + 1 < g.W;
    const T* zero = reinterpret_cast<const T*>(g_zero_slice);
    const T* p00 = img + (h0 * g.W + w0) * g.C;
    cell.c[0] = (y0 && x0) ? p00 : zero;
    cell.c[1] = (y0 && x1) ? p00 + g.C : zero;
    cell.c[2] = (y1 && x0) ? p00 + g.W * g.C : zero;
    cell.c[3] = (y1 && x1) ? p00 + g.W * g.C + g.C : zero;
    return cell;
}

}  // namespace dcn4

// Host-side launchers (defined in dcn4_forward.cu / dcn4_backward.cu).
namespace dcn4 {
cudaError_t launch_forward(const Geometry& g, int dtype, const void* value, const void* om, void* out,
                           cudaStream_t stream);
// grad_offset_mask and the per-image reach (int[N], pre-filled with -1).
// Also writes the per-sample entries of `sa` and the bounding box of each
// output pixel's cells, boxes[N, Ho, Wo].
cudaError_t launch_backward_samples(const Geometry& g, int dtype, const void* value, const void* om,
                                    const void* gout, void* gom, int* reach, SampleArrays sa, uint32_t* boxes,
                                    cudaStream_t stream);
// grad_value from the reach, sample entries and boxes written by launch_backward_samples.
cudaError_t launch_backward_value(const Geometry& g, int dtype, const void* om, const void* gout, void* gvalue,
                                  const int* reach, SampleArrays sa, const uint32_t* boxes,
                                  cudaStream_t stream);
// Points a grad_offset_mask CTA stages before filing them: all K for the 3x3
// grids (compiled unrolled), chunks of 8 for the generic grids.
__host__ __device__ inline int filing_chunk(const Geometry& g) { return (g.kh == 3 && g.kw == 3) ? g.K : (g.K < 8 ? g.K : 8); }
// Threads of one grad_offset_mask CTA: whole warps (the kernel shuffles).
inline int samples_threads(const Geometry& g) { return (g.pix_per_cta * g.G * g.nslice + 31) / 32 * 32; }
// Dynamic shared memory bytes of one CTA.
size_t forward_smem_bytes(const Geometry& g, int elem_bytes);
// Forward with the linear producer (16-bit dtypes): offset_mask = x W^T + b per
// tile, x [N, Ho, Wo, Cx], w [P, Cx], b [P] or null, om_out [N, Ho, Wo, P] or null.
cudaError_t launch_forward_linear(const Geometry& g, int dtype, const void* value, const void* x, const void* w,
                                  const void* b, void* out, void* om_out, int Cx, cudaStream_t stream);
// mode 0: mma.sync, W read from global memory; 1: mma.sync, W staged in shared
// memory; 2: tcgen05 (W and the x tiles swizzled in shared memory).
size_t forward_linear_smem_bytes(const Geometry& g, int Cx, int mode);
// The fused forward's producer mode for this shape.
int forward_linear_mode(const Geometry& g, int Cx);
// Forward with the output projection behind the sampler (16-bit dtypes): out =
// core W^T + b per tile, w [Cout, C], b [Cout] or null, core_out [N, Ho, Wo, C]
// or null.  Shapes: 16-, 32- or 64-pixel tiles, C a multiple of 64 up to 256,
// Cout a multiple of 16 up to 128 (forward_proj_shape_ok).
bool forward_proj_shape_ok(const Geometry& g, int Cout);
size_t forward_proj_smem_bytes(const Geometry& g, int Cout);
cudaError_t launch_forward_proj(const Geometry& g, int dtype, const void* value, const void* om, const void* w,
                                const void* b, void* out, void* core_out, int Cout, cudaStream_t stream);
// The status word of the forward's tcgen05 paths (producer and projection):
// nonzero once a bounded wait gave up.  Synchronous; reset clears it.
cudaError_t forward_tc_status(unsigned* status, bool reset);
// Gradients of the linear producer from gom = grad_offset_mask as an [M, P]
// matrix (16-bit dtypes): gx = gom W [M, Cx], gw = gom^T x [P, Cx], gb = column
// sums of gom [P]; any of the three may be null.  ws: fp32 scratch of
// linear_backward_workspace_bytes(P, Cx) bytes (grad_W and grad_b accumulators).
size_t linear_backward_workspace_bytes(int P, int Cx);
cudaError_t launch_linear_backward(int dtype, long long M, int P, int Cx, const void* x, const void* w,
                                   const void* gom, void* gx, void* gw, void* gb, float* ws, cudaStream_t stream);
size_t backward_smem_bytes(const Geometry& g, int elem_bytes);
// Single-scale deformable attention (dcn4_attn.cu): g holds the value map (N, H,
// W, G, Cg, C), the points per query (K), the row length (P), offset_scale (s)
// and the slice split (vec, nslice); Nq queries per image.  The backward
// accumulates grad_value in fp32 at `acc` (grad_value itself for fp32 I/O,
// zeroed by the caller) and rounds it into gvalue for 16-bit I/O.
size_t attn_smem_bytes(const Geometry& g, int elem_bytes, bool backward);
cudaError_t launch_attn_forward(const Geometry& g, int dtype, int Nq, const void* value, const float* ref,
                                const void* ol, void* out, cudaStream_t stream);
cudaError_t launch_attn_backward(const Geometry& g, int dtype, int Nq, const void* value, const float* ref,
                                 const void* ol, const void* gout, void* gvalue, void* gol, float* acc,
                                 cudaStream_t stream);
size_t backward_value_smem_bytes(const Geometry& g);
}  // namespace dcn4
