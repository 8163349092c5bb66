// dcn4_backward.cu — gradients of the DCNv4 core spatial aggregation.
//
// For every sample (output pixel p, group g, point k) with location
// (h, w) = anchor + s*(dy, dx), bilinear cell corners v_ab and weights
// w_ab = (a ? lh : 1-lh)(b ? lw : 1-lw), and gy = grad_out of (p, g):
//   d/d m_k   = <gy, S>,                        S = sum_ab w_ab v_ab
//   d/d dx_k  = s * m_k * <gy, dS/dw>,          dS/dw = (1-lh)(v01 - v00) + lh(v11 - v10)
//   d/d dy_k  = s * m_k * <gy, dS/dh>,          dS/dh = (1-lw)(v10 - v00) + lw(v11 - v01)
//   grad_value[corner ab] += m_k * w_ab * gy     (every in-image corner)
// where <.,.> sums over the group's C' channels.
//
// Two kernels, no atomics on gradient data:
//
// samples_kernel (output tiles, the forward's mapping).  The three per-sample
//   gradients follow from the four per-corner dot products d_ab = <gy, v_ab>:
//   each corner slice is gathered once (256-bit load), dotted with gy in fp32,
//   reduced over the threads sharing the group, and the grad_offset_mask rows
//   (padding tail = 0) are assembled in shared memory and stored once.  It
//   also records, per image, the reach R: the largest distance (per
//   coordinate, in pixels) between a grid anchor and a corner of a cell that
//   touches the image; and, per sample, a 2-byte code of its cell relative to
//   its anchor.
//
// value_kernel (input tiles).  grad_value is pulled, not scattered: a CTA owns
//   a BH x BW tile of input pixels (all groups) and writes each of their
//   grad_value elements exactly once.  The samples that can touch the tile come
//   from output pixels whose anchors lie within R of it; the CTA reads those
//   samples' cell codes, re-forms the locations of the ones whose cell touches
//   the tile (the same fp32 fma as the forward, so the same cells), and
//   counting-sorts them by (group, cell) in
//   shared memory, then each thread sums m * w_ab * gy over the samples of the
//   four cells its pixel is a corner of.  Should the sorted samples not fit in
//   shared memory (a pathological concentration of samples), the CTA falls
//   back to having each thread scan the candidate samples directly: slower,
//   same result.
#include <type_traits>

#include "dcn4_common.cuh"

namespace dcn4 {
namespace {

__device__ __forceinline__ int floor_div(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }
__device__ __forceinline__ int ceil_div(int a, int b) { return -floor_div(-a, b); }

// <gy, the VEC x 16 bytes of channels at src>, in fp32.
template <typename T, int VEC>
__device__ __forceinline__ float corner_dot(const float2* gy, const T* src) {
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

// gy (this thread's VEC x 16 bytes of grad_out channels) as fp32 pairs.
template <typename T, int VEC>
__device__ __forceinline__ void load_gy(float2* gy, const T* src) {
    constexpr int HALF = Elem<T>::per16 / 2;
    uint4 raw[VEC];
    if constexpr (VEC == 2) {
        ld_gather32(src, raw[0], raw[1]);
    } else {
        raw[0] = ld_gather(src);
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) unpack(raw[v], gy + v * HALF, T());
}

// Cell code of a sample: the offset of its cell's top-left corner from the
// grid anchor, (row, column) as two int8 (low byte = row).  A sample that
// touches no pixel is kCodeNone.  Offsets beyond +-126 are clamped: the
// grad_value pass only trusts codes for images whose reach is at most 126.
constexpr uint16_t kCodeNone = 0x8080;
constexpr int kCodeReach = 126;
// Candidate output pixels a grad_value CTA lists in shared memory (beyond that
// it walks its whole candidate window instead).
constexpr int kListCap = 2048;

__device__ __forceinline__ uint16_t cell_code(bool any, int dh, int dw) {
    if (!any) return kCodeNone;
    dh = min(127, max(-127, dh));
    dw = min(127, max(-127, dw));
    return static_cast<uint16_t>((dh & 0xff) | ((dw & 0xff) << 8));
}

// Per-sample entry the sample pass leaves for the grad_value pass.  fp32 I/O:
// the 2-byte cell code (the grad_value pass re-forms the exact weights from
// the offsets).  16-bit I/O: an 8-byte record — cell code, the mask's own 16
// bits, lh and lw as 16-bit fixed point — so the grad_value pass never reads
// the offsets.
template <typename T>
using SampleEntry = std::conditional_t<sizeof(T) == 2, uint64_t, uint16_t>;

__device__ __forceinline__ uint32_t fix16(float f) { return min(65535u, static_cast<uint32_t>(f * 65536.f + 0.5f)); }

template <typename T>
__device__ __forceinline__ uint16_t raw_bits(T x) {
    uint16_t b;
    memcpy(&b, &x, 2);
    return b;
}

// Grid cell (ih, iw) of sampling point k (columns outer, rows inner, centre
// skipped when remove_center is set).
__device__ __forceinline__ void grid_cell_of(const Geometry& g, int k, int& ih, int& iw) {
    int idx = k;
    if (g.remove_center) {
        const int centre = (g.kw / 2) * g.kh + g.kh / 2;
        if (idx >= centre) ++idx;
    }
    iw = idx / g.kh;
    ih = idx - iw * g.kh;
}

// ---------------------------------------------------------------------------
// grad_offset_mask + reach
// ---------------------------------------------------------------------------
template <typename T, int VEC, int KH, int KW, bool RC>
__global__ void __launch_bounds__(256) samples_kernel(const Geometry g, const T* __restrict__ value,
                                                      const T* __restrict__ om, const T* __restrict__ gout,
                                                      T* __restrict__ gom, int* __restrict__ reach,
                                                      void* __restrict__ codes, uint32_t* __restrict__ boxes) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_reach;
    __shared__ int s_box[4 * 256];  // per tile pixel: min/max cell row, min/max cell column (relative)
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    const int tile_elems = g.TH * g.TW * g.P;
    T* om_s = reinterpret_cast<T*>(smem);
    T* gom_s = reinterpret_cast<T*>(smem + tile_elems * sizeof(T));  // P % 8 == 0 keeps this 16-byte aligned

    const Tile t = tile_of_block(g);
    stage_tile_rows(om_s, om, g, t);
    for (int i = threadIdx.x; i < tile_elems; i += blockDim.x) gom_s[i] = static_cast<T>(0.f);
    for (int i = threadIdx.x; i < g.TH * g.TW; i += blockDim.x) {
        s_box[4 * i] = 127;
        s_box[4 * i + 1] = -128;
        s_box[4 * i + 2] = 127;
        s_box[4 * i + 3] = -128;
    }
    if (threadIdx.x == 0) s_reach = -1;
    __syncthreads();

    const int lanes_pp = g.G * g.nslice;
    const int lp = threadIdx.x / lanes_pp;
    const int py = lp / g.TW;
    const int px = lp - py * g.TW;
    // Threads past the tile edge stay in the loop (their samples touch
    // nothing) so that every lane of a warp reaches the shuffles.
    const bool active = py < t.th && px < t.tw;
    const int r = threadIdx.x - lp * lanes_pp;
    const int grp = r / g.nslice;
    const int sl = r - grp * g.nslice;
    const int ho = t.ho0 + (active ? py : 0), wo = t.wo0 + (active ? px : 0);
    const int lrow = (active ? lp : 0) * g.P + grp * 3 * (KH > 0 ? KH * KW - (RC ? 1 : 0) : g.K);

    const int K = KH > 0 ? KH * KW - (RC ? 1 : 0) : g.K;
    const int kh = KH > 0 ? KH : g.kh;
    const int kw = KW > 0 ? KW : g.kw;
    const bool rc = KH > 0 ? RC : g.remove_center != 0;
    const T* row = om_s + lrow;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* img = value + static_cast<long long>(t.n) * g.H * g.W * g.C + ch_off;
    const int hb = ho * g.sh - g.ph, wb = wo * g.sw - g.pw;

    float2 gy[PAIRS];
    const long long pix = (static_cast<long long>(t.n) * g.Ho + ho) * g.Wo + wo;
    load_gy<T, VEC>(gy, gout + pix * g.C + ch_off);
    SampleEntry<T>* code = static_cast<SampleEntry<T>*>(codes) + (pix * g.G + grp) * K;  // [N, Ho, Wo, G, K]
    const bool writer = active && sl == 0;
    int my_reach = -1;
    int bmin_h = 127, bmax_h = -128, bmin_w = 127, bmax_w = -128;  // cells relative to (hb, wb)

    int k = 0;
#pragma unroll
    for (int iw = 0; iw < kw; ++iw) {
        const int aw = wb + iw * g.dw;  // anchor column
#pragma unroll
        for (int ih = 0; ih < kh; ++ih) {
            if (rc && iw == kw / 2 && ih == kh / 2) continue;
            const int kk = k++;
            const int ah = hb + ih * g.dh;  // anchor row
            const float dx = to_f32(row[2 * kk]);
            const float dy = to_f32(row[2 * kk + 1]);
            const float m = to_f32(row[2 * K + kk]);
            const float h = active ? __fmaf_rn(g.s, dy, static_cast<float>(ah)) : -2.f;
            const float w = __fmaf_rn(g.s, dx, static_cast<float>(aw));
            const Cell<T> cell = bilinear_cell(g, img, h, w);
            float d00 = corner_dot<T, VEC>(gy, cell.c[0]);
            float d01 = corner_dot<T, VEC>(gy, cell.c[1]);
            float d10 = corner_dot<T, VEC>(gy, cell.c[2]);
            float d11 = corner_dot<T, VEC>(gy, cell.c[3]);
            for (int off = g.nslice >> 1; off > 0; off >>= 1) {
                d00 += __shfl_xor_sync(0xffffffffu, d00, off);
                d01 += __shfl_xor_sync(0xffffffffu, d01, off);
                d10 += __shfl_xor_sync(0xffffffffu, d10, off);
                d11 += __shfl_xor_sync(0xffffffffu, d11, off);
            }
            if (cell.any) {
                if (sl == 0) {
                    const float hl = 1.f - cell.lh, wl = 1.f - cell.lw;
                    const float sm = g.s * m;
                    T* gr = gom_s + lrow;  // rounded once, to the I/O dtype
                    gr[2 * kk] = from_f32<T>(sm * (hl * (d01 - d00) + cell.lh * (d11 - d10)));
                    gr[2 * kk + 1] = from_f32<T>(sm * (wl * (d10 - d00) + cell.lw * (d11 - d01)));
                    gr[2 * K + kk] = from_f32<T>(hl * (wl * d00 + cell.lw * d01) + cell.lh * (wl * d10 + cell.lw * d11));
                }
                const int dh = max(abs(cell.h0 - ah), abs(cell.h0 + 1 - ah));
                const int dw = max(abs(cell.w0 - aw), abs(cell.w0 + 1 - aw));
                my_reach = max(my_reach, max(dh, dw));
                bmin_h = min(bmin_h, cell.h0 - hb);
                bmax_h = max(bmax_h, cell.h0 - hb);
                bmin_w = min(bmin_w, cell.w0 - wb);
                bmax_w = max(bmax_w, cell.w0 - wb);
            }
            if (writer) {
                const uint16_t cd = cell_code(cell.any, cell.h0 - ah, cell.w0 - aw);
                if constexpr (sizeof(T) == 2) {
                    code[kk] = static_cast<uint64_t>(cd) | (static_cast<uint64_t>(raw_bits(row[2 * K + kk])) << 16) |
                               (static_cast<uint64_t>(fix16(cell.lh)) << 32) | (static_cast<uint64_t>(fix16(cell.lw)) << 48);
                } else {
                    code[kk] = cd;
                }
            }
        }
    }

    for (int off = 16; off > 0; off >>= 1) my_reach = max(my_reach, __shfl_xor_sync(0xffffffffu, my_reach, off));
    if ((threadIdx.x & 31) == 0 && my_reach >= 0) atomicMax(&s_reach, my_reach);
    if (writer && bmax_h >= bmin_h) {
        atomicMin(&s_box[4 * lp], max(-127, bmin_h));
        atomicMax(&s_box[4 * lp + 1], min(127, bmax_h));
        atomicMin(&s_box[4 * lp + 2], max(-127, bmin_w));
        atomicMax(&s_box[4 * lp + 3], min(127, bmax_w));
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_reach >= 0) atomicMax(reach + t.n, s_reach);
    for (int i = threadIdx.x; i < t.th * g.TW; i += blockDim.x) {
        const int r2 = i / g.TW, c2 = i - r2 * g.TW;
        if (c2 >= t.tw) continue;
        const long long bp = (static_cast<long long>(t.n) * g.Ho + t.ho0 + r2) * g.Wo + t.wo0 + c2;
        boxes[bp] = (s_box[4 * i] & 0xff) | ((s_box[4 * i + 1] & 0xff) << 8) | ((s_box[4 * i + 2] & 0xff) << 16) |
                    (static_cast<uint32_t>(s_box[4 * i + 3] & 0xff) << 24);
    }

    // grad_offset_mask rows of the tile, 16-byte stores.
    const int row_vecs = t.tw * g.P / EPV;
    for (int i = threadIdx.x; i < t.th * row_vecs; i += blockDim.x) {
        const int rr = i / row_vecs;
        const int c = i - rr * row_vecs;
        const long long grow = (static_cast<long long>(t.n) * g.Ho + t.ho0 + rr) * g.Wo + t.wo0;
        st_global(gom + grow * g.P + c * EPV, *reinterpret_cast<const uint4*>(gom_s + rr * g.TW * g.P + c * EPV));
    }
}

// ---------------------------------------------------------------------------
// grad_value (pull over a counting sort of the samples touching the tile)
// ---------------------------------------------------------------------------

// acc += wt * gy slice at src.
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

// One candidate sample of the tile scan: the cell it falls in.
struct Candidate {
    int h0, w0;
    float lh, lw;
    bool any;
};

template <typename T>
__device__ __forceinline__ float ld_stream_elem(const T* p) {
    if constexpr (sizeof(T) == 2) {
        const uint16_t b = ld_stream_u16(p);
        T x;
        memcpy(&x, &b, 2);
        return to_f32(x);
    } else {
        float x;
        asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(x) : "l"(p));
        return x;
    }
}

template <typename T>
__device__ __forceinline__ Candidate candidate(const Geometry& g, const T* om_row, int k, int ho, int wo, int ih,
                                               int iw) {
    const float dx = ld_stream_elem(om_row + 2 * k);
    const float dy = ld_stream_elem(om_row + 2 * k + 1);
    const float h = __fmaf_rn(g.s, dy, static_cast<float>(ho * g.sh - g.ph + ih * g.dh));
    const float w = __fmaf_rn(g.s, dx, static_cast<float>(wo * g.sw - g.pw + iw * g.dw));
    Candidate c;
    c.any = h >= -1.f && h < static_cast<float>(g.H) && w >= -1.f && w < static_cast<float>(g.W);
    const float hc = c.any ? h : 0.f, wc = c.any ? w : 0.f;
    const float h0f = floorf(hc), w0f = floorf(wc);
    c.lh = hc - h0f;
    c.lw = wc - w0f;
    c.h0 = static_cast<int>(h0f);
    c.w0 = static_cast<int>(w0f);
    return c;
}

// Sample records of the grad_value sort.  Wide (16 bytes, fp32 I/O): image
// pixel index of p, m(1-lh), m lh, lw.  Compact (8 bytes, 16-bit I/O): index of
// p in the CTA's candidate list, the mask's own 16 bits, and lh, lw as 16-bit
// fixed point (error below 2^-17, far under the I/O rounding).
__device__ __forceinline__ float from_bits(uint16_t b, __half) {
    __half h;
    memcpy(&h, &b, 2);
    return __half2float(h);
}
__device__ __forceinline__ float from_bits(uint16_t b, __nv_bfloat16) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

template <typename T, int VEC, bool COMPACT>
__global__ void __launch_bounds__(512, 2) value_kernel(const Geometry g, const T* __restrict__ om,
                                                       const T* __restrict__ gout, T* __restrict__ gvalue,
                                                       const int* __restrict__ reach,
                                                       const void* __restrict__ codes,
                                                       const uint32_t* __restrict__ boxes) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_warp[32];
    __shared__ int s_total;
    __shared__ int s_nlist;
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;

    // Input tile of this CTA.
    const int per_img = g.btiles_h * g.btiles_w;
    const int n = blockIdx.x / per_img;
    const int tr = blockIdx.x - n * per_img;
    const int by = tr / g.btiles_w;
    const int y0 = by * g.BH, x0 = (tr - by * g.btiles_w) * g.BW;
    const int bh = min(g.BH, g.H - y0), bw = min(g.BW, g.W - x0);
    const int cells_w = g.BW + 1;
    const int cells = (g.BH + 1) * cells_w;
    const int nbins = g.G * cells;
    int* cnt = reinterpret_cast<int*>(smem);
    int* cur = cnt + nbins;
    uint32_t* s_list = reinterpret_cast<uint32_t*>(cur + nbins);  // candidate pixels: (ho << 16) | wo
    unsigned char* rec_base = smem + ((2 * nbins + kListCap) * sizeof(int) + 15) / 16 * 16;
    float4* rec_w = reinterpret_cast<float4*>(rec_base);
    uint2* rec_c = reinterpret_cast<uint2*>(rec_base);

    // Samples that can touch the tile come from output pixels whose anchor
    // (for the sample's grid point) lies within R of the tile.
    const int R = reach[n];
    const int GK = g.G * g.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const bool use_codes = R <= kCodeReach;  // else cells are re-formed from the offsets
    const bool boxes_exact = use_codes && R + max((g.kh - 1) * g.dh, (g.kw - 1) * g.dw) <= 127;
    int ho_lo = 0, ho_hi = -1, wo_lo = 0, wo_hi = -1;
    if (R >= 0) {
        ho_lo = max(0, ceil_div(y0 - R + g.ph - (g.kh - 1) * g.dh, g.sh));
        ho_hi = min(g.Ho - 1, floor_div(y0 + bh - 1 + R + g.ph, g.sh));
        wo_lo = max(0, ceil_div(x0 - R + g.pw - (g.kw - 1) * g.dw, g.sw));
        wo_hi = min(g.Wo - 1, floor_div(x0 + bw - 1 + R + g.pw, g.sw));
    }
    const int e_w = max(0, wo_hi - wo_lo + 1);
    const int e_cnt = e_w * max(0, ho_hi - ho_lo + 1);
    const long long pix0 = static_cast<long long>(n) * g.Ho * g.Wo;

    if (threadIdx.x == 0) s_nlist = 0;
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) cnt[i] = 0;
    __syncthreads();

    // List the candidate pixels whose cell bounding box meets the tile's cells.
    if (boxes_exact) {
        for (int e0 = warp * 32; e0 < e_cnt; e0 += nwarps * 32) {
            const int e = e0 + lane;
            bool keep = false;
            int ho = 0, wo = 0;
            if (e < e_cnt) {
                const int eh = e / e_w;
                ho = ho_lo + eh;
                wo = wo_lo + (e - eh * e_w);
                const uint32_t box = boxes[pix0 + static_cast<long long>(ho) * g.Wo + wo];
                const int bh0 = ho * g.sh - g.ph, bw0 = wo * g.sw - g.pw;
                const int rmin = bh0 + static_cast<int8_t>(box & 0xff), rmax = bh0 + static_cast<int8_t>((box >> 8) & 0xff);
                const int cmin = bw0 + static_cast<int8_t>((box >> 16) & 0xff), cmax = bw0 + static_cast<int8_t>(box >> 24);
                keep = rmax >= y0 - 1 && rmin <= y0 + bh - 1 && cmax >= x0 - 1 && cmin <= x0 + bw - 1;
            }
            const unsigned ball = __ballot_sync(0xffffffffu, keep);
            int base = 0;
            if (lane == 0 && ball) base = atomicAdd(&s_nlist, __popc(ball));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int pos = base + __popc(ball & ((1u << lane) - 1));
            if (keep && pos < kListCap) s_list[pos] = (static_cast<uint32_t>(ho) << 16) | static_cast<uint32_t>(wo);
        }
    }
    __syncthreads();
    const bool listed = boxes_exact && s_nlist <= kListCap && g.Ho <= 65535 && g.Wo <= 65535;
    const int nlist = s_nlist;

    // Scan mapping: each thread keeps one (group, point) and walks the listed
    // pixels (or, without a list, every pixel whose anchor for that point is
    // within R of the tile), a slot of pixels at a time.
    const int spt = blockDim.x / GK;
    const int tslot = threadIdx.x / GK;
    const int gk = threadIdx.x - tslot * GK;
    const bool scanner = tslot < spt;
    const int sg = gk / g.K;
    const int sk = gk - sg * g.K;
    int s_ih, s_iw;
    grid_cell_of(g, sk, s_ih, s_iw);
    const int ah0 = s_ih * g.dh - g.ph, aw0 = s_iw * g.dw - g.pw;  // anchor = (ho*sh + ah0, wo*sw + aw0)
    int kh_lo = 0, kh_hi = -1, kw_lo = 0, kw_hi = -1;
    if (R >= 0) {
        kh_lo = max(0, ceil_div(y0 - R - ah0, g.sh));
        kh_hi = min(g.Ho - 1, floor_div(y0 + bh - 1 + R - ah0, g.sh));
        kw_lo = max(0, ceil_div(x0 - R - aw0, g.sw));
        kw_hi = min(g.Wo - 1, floor_div(x0 + bw - 1 + R - aw0, g.sw));
    }
    const int k_w = max(0, kw_hi - kw_lo + 1);
    const int k_cnt = listed ? nlist : k_w * max(0, kh_hi - kh_lo + 1);
    const SampleEntry<T>* code_n = static_cast<const SampleEntry<T>*>(codes) + pix0 * GK + gk;
    const T* om_n = om + pix0 * g.P + sg * 3 * g.K;

    // Pass 0 counts the samples of each (group, cell); pass 1 places their records in bin order.
    bool sorted = true;
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
            // Exclusive scan of the counts -> cursors (block-wide, thread-contiguous chunks).
            const int per = (nbins + blockDim.x - 1) / blockDim.x;
            const int b0 = threadIdx.x * per;
            int local = 0;
            for (int b = b0; b < min(nbins, b0 + per); ++b) local += cnt[b];
            int incl = local;
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (lane == 31) s_warp[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                int v = lane < nwarps ? s_warp[lane] : 0;
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += u;
                }
                if (lane < nwarps) s_warp[lane] = v;  // inclusive warp totals
                if (lane == nwarps - 1) s_total = v;
            }
            __syncthreads();
            int run = incl - local + (warp > 0 ? s_warp[warp - 1] : 0);
            for (int b = b0; b < min(nbins, b0 + per); ++b) {
                cur[b] = run;
                run += cnt[b];
            }
            __syncthreads();
            sorted = s_total <= g.bcap;
            if (!sorted) break;
        }
        if (scanner && listed) {
            // Lean walk over the listed pixels: 32-bit math, constants hoisted.
            const int Wo = g.Wo, sh = g.sh, sw = g.sw;
            const int hbase = ah0 - (y0 - 1), wbase = aw0 - (x0 - 1);  // cell row/col relative to the tile's cells
            const int binbase = sg * cells;
            for (int e = tslot; e < nlist; e += spt) {
                const uint32_t lv = s_list[e];
                const int ho = static_cast<int>(lv >> 16), wo = static_cast<int>(lv & 0xffff);
                const int pix = ho * Wo + wo;
                SampleEntry<T> sr;
                if constexpr (COMPACT) {
                    sr = ld_stream_u64(code_n + static_cast<long long>(pix) * GK);
                } else {
                    sr = ld_stream_u16(code_n + static_cast<long long>(pix) * GK);
                }
                const uint16_t cd = static_cast<uint16_t>(sr & 0xffff);
                const int ch = ho * sh + hbase + static_cast<int8_t>(cd & 0xff);
                const int cw = wo * sw + wbase + static_cast<int8_t>(cd >> 8);
                if (cd == kCodeNone || static_cast<unsigned>(ch) > static_cast<unsigned>(bh) ||
                    static_cast<unsigned>(cw) > static_cast<unsigned>(bw))
                    continue;
                const int bin = binbase + ch * cells_w + cw;
                if (pass == 0) {
                    atomicAdd(&cnt[bin], 1);
                } else {
                    const int slot = atomicAdd(&cur[bin], 1);
                    if constexpr (COMPACT) {
                        // the sample pass already left the mask bits and fixed-point lh, lw
                        rec_c[slot] = make_uint2(static_cast<uint32_t>(e) | (static_cast<uint32_t>(sr) & 0xffff0000u),
                                                 static_cast<uint32_t>(sr >> 32));
                    } else {
                        const T* orow = om_n + static_cast<long long>(pix) * g.P;
                        const Candidate c = candidate(g, orow, sk, ho, wo, s_ih, s_iw);
                        const float mf = ld_stream_elem(orow + 2 * g.K + sk);
                        const float b = mf * c.lh;
                        rec_w[slot] = make_float4(__int_as_float(pix), mf - b, b, c.lw);
                    }
                }
            }
        } else if (scanner) {
            // Without a list: every pixel whose anchor for this point lies within R.
            int ho = 0, wo = 0;
            if (tslot < k_cnt) {
                const int eh = tslot / k_w;
                ho = kh_lo + eh;
                wo = kw_lo + tslot - eh * k_w;
            }
            for (int e = tslot; e < k_cnt; e += spt) {
                const long long pix = static_cast<long long>(ho) * g.Wo + wo;
                int h0, w0;
                bool any;
                Candidate c;
                if (use_codes) {
                    uint16_t cd;
                    if constexpr (COMPACT) {
                        cd = static_cast<uint16_t>(ld_stream_u64(code_n + pix * GK) & 0xffff);
                    } else {
                        cd = ld_stream_u16(code_n + pix * GK);
                    }
                    any = cd != kCodeNone;
                    h0 = ho * g.sh + ah0 + static_cast<int8_t>(cd & 0xff);
                    w0 = wo * g.sw + aw0 + static_cast<int8_t>(cd >> 8);
                } else {
                    c = candidate(g, om_n + pix * g.P, sk, ho, wo, s_ih, s_iw);
                    any = c.any;
                    h0 = c.h0;
                    w0 = c.w0;
                }
                const int ch = h0 - (y0 - 1), cw = w0 - (x0 - 1);
                if (any && static_cast<unsigned>(ch) <= static_cast<unsigned>(bh) &&
                    static_cast<unsigned>(cw) <= static_cast<unsigned>(bw)) {
                    const int bin = sg * cells + ch * cells_w + cw;
                    if (pass == 0) {
                        atomicAdd(&cnt[bin], 1);
                    } else if constexpr (!COMPACT) {  // compact records need the list (direct path instead)
                        const T* orow = om_n + pix * g.P;
                        if (use_codes) c = candidate(g, orow, sk, ho, wo, s_ih, s_iw);
                        const int slot = atomicAdd(&cur[bin], 1);
                        const float mf = ld_stream_elem(orow + 2 * g.K + sk);
                        const float b = mf * c.lh;
                        rec_w[slot] = make_float4(__int_as_float(static_cast<int>(pix)), mf - b, b, c.lw);
                    }
                }
                wo += spt;  // next pixel of this slot
                while (wo > kw_hi) {
                    wo -= k_w;
                    ++ho;
                }
            }
        }
        __syncthreads();
    }
    // Compact records need the list; without it the tile takes the direct path.
    if (COMPACT && !listed) sorted = false;

    // Pull: thread -> (input pixel q of the tile, group, slice).
    const int lanes_pp = g.G * g.nslice;
    const int q = threadIdx.x / lanes_pp;
    const int qy = q / g.BW, qx = q - (q / g.BW) * g.BW;
    if (q >= g.BH * g.BW || qy >= bh || qx >= bw) return;
    const int rr = threadIdx.x - q * lanes_pp;
    const int grp = rr / g.nslice;
    const int sl = rr - grp * g.nslice;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* gy_img = gout + pix0 * g.C + ch_off;

    float2 acc[PAIRS];
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) acc[i] = make_float2(0.f, 0.f);

    if (sorted) {
        // q is corner (a, b) of the cell with top-left (qy - a, qx - b).
#pragma unroll
        for (int a = 0; a < 2; ++a) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int bin = grp * cells + (qy - a + 1) * cells_w + (qx - b + 1);
                const int end = cur[bin];
                int j = end - cnt[bin];
                // Two records per step, so two grad_out gathers are in flight.
                for (; j + 1 < end; j += 2) {
                    const T* src[2];
                    float wt[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if constexpr (COMPACT) {
                            const uint2 r = rec_c[j + u];
                            const uint32_t lv = s_list[r.x & 0xffff];
                            const float m = from_bits(static_cast<uint16_t>(r.x >> 16), T());
                            const float hq = static_cast<float>(a ? (r.y & 0xffff) : 65536u - (r.y & 0xffff));
                            const float wq = static_cast<float>(b ? (r.y >> 16) : 65536u - (r.y >> 16));
                            wt[u] = m * (hq * wq) * 0x1p-32f;
                            src[u] = gy_img + ((lv >> 16) * static_cast<long long>(g.Wo) + (lv & 0xffff)) * g.C;
                        } else {
                            const float4 r = rec_w[j + u];
                            wt[u] = (a ? r.z : r.y) * (b ? r.w : 1.f - r.w);
                            src[u] = gy_img + static_cast<long long>(__float_as_int(r.x)) * g.C;
                        }
                    }
                    uint4 raw[2][VEC];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if constexpr (VEC == 2) {
                            ld_keep32(src[u], raw[u][0], raw[u][1]);
                        } else {
                            raw[u][0] = ld_keep16(src[u]);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float2 w2 = make_float2(wt[u], wt[u]);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            float2 f[EPV / 2];
                            unpack(raw[u][v], f, T());
#pragma unroll
                            for (int i = 0; i < EPV / 2; ++i)
                                acc[v * (EPV / 2) + i] = __ffma2_rn(w2, f[i], acc[v * (EPV / 2) + i]);
                        }
                    }
                }
                if (j < end) {
                    const T* src;
                    float wt;
                    if constexpr (COMPACT) {
                        const uint2 r = rec_c[j];
                        const uint32_t lv = s_list[r.x & 0xffff];
                        const float m = from_bits(static_cast<uint16_t>(r.x >> 16), T());
                        const float hq = static_cast<float>(a ? (r.y & 0xffff) : 65536u - (r.y & 0xffff));
                        const float wq = static_cast<float>(b ? (r.y >> 16) : 65536u - (r.y >> 16));
                        wt = m * (hq * wq) * 0x1p-32f;
                        src = gy_img + ((lv >> 16) * static_cast<long long>(g.Wo) + (lv & 0xffff)) * g.C;
                    } else {
                        const float4 r = rec_w[j];
                        wt = (a ? r.z : r.y) * (b ? r.w : 1.f - r.w);
                        src = gy_img + static_cast<long long>(__float_as_int(r.x)) * g.C;
                    }
                    accumulate<T, VEC>(acc, src, wt);
                }
            }
        }
    } else {
        // Direct path: scan every candidate sample of this group.
        const int uh_lo = max(0, ceil_div(y0 - R + g.ph - (g.kh - 1) * g.dh, g.sh));
        const int uh_hi = min(g.Ho - 1, floor_div(y0 + bh - 1 + R + g.ph, g.sh));
        const int uw_lo = max(0, ceil_div(x0 - R + g.pw - (g.kw - 1) * g.dw, g.sw));
        const int uw_hi = min(g.Wo - 1, floor_div(x0 + bw - 1 + R + g.pw, g.sw));
        const int u_w = max(0, uw_hi - uw_lo + 1);
        const int u_cnt = R >= 0 ? u_w * max(0, uh_hi - uh_lo + 1) : 0;
        const int gy_abs = y0 + qy, gx_abs = x0 + qx;
        const T* om_g = om + pix0 * g.P + grp * 3 * g.K;
        for (int e = 0; e < u_cnt; ++e) {
            const int eh = e / u_w;
            const int ho = uh_lo + eh, wo = uw_lo + (e - eh * u_w);
            const T* orow = om_g + static_cast<long long>(ho * g.Wo + wo) * g.P;
            for (int k = 0; k < g.K; ++k) {
                int ih, iw;
                grid_cell_of(g, k, ih, iw);
                const Candidate c = candidate(g, orow, k, ho, wo, ih, iw);
                const int a = gy_abs - c.h0, b = gx_abs - c.w0;
                if (c.any && a >= 0 && a <= 1 && b >= 0 && b <= 1) {
                    const float m = to_f32(orow[2 * g.K + k]);
                    const float wt = m * (a ? c.lh : 1.f - c.lh) * (b ? c.lw : 1.f - c.lw);
                    accumulate<T, VEC>(acc, gy_img + static_cast<long long>(ho * g.Wo + wo) * g.C, wt);
                }
            }
        }
    }

    T* dst = gvalue + ((static_cast<long long>(n) * g.H + y0 + qy) * g.W + x0 + qx) * g.C + ch_off;
    if constexpr (VEC == 2) {
        st_global32(dst, pack(acc, T()), pack(acc + EPV / 2, T()));
    } else {
        st_global(dst, pack(acc, T()));
    }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------

// Opt the kernel in to `smem` bytes of dynamic shared memory (needed whenever
// static + dynamic exceed the 48 KB default).
template <typename Kern>
cudaError_t allow_smem(Kern kern, size_t smem) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
}

template <typename T, int VEC, int KH, int KW, bool RC>
cudaError_t launch_samples_typed(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                                 int* reach, void* codes, uint32_t* boxes, cudaStream_t stream) {
    const size_t smem = backward_smem_bytes(g, sizeof(T));
    auto kern = samples_kernel<T, VEC, KH, KW, RC>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const long long blocks = static_cast<long long>(g.N) * g.tiles_h * g.tiles_w;
    const int threads = (g.pix_per_cta * g.G * g.nslice + 31) / 32 * 32;  // whole warps (shuffles)
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(g, static_cast<const T*>(value),
                                                                   static_cast<const T*>(om), static_cast<const T*>(gout),
                                                                   static_cast<T*>(gom), reach, codes, boxes);
    return cudaGetLastError();
}

template <typename T, int VEC>
cudaError_t launch_samples_grid(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                                int* reach, void* codes, uint32_t* boxes, cudaStream_t stream) {
    if (g.kh == 3 && g.kw == 3) {
        return g.remove_center
                   ? launch_samples_typed<T, VEC, 3, 3, true>(g, value, om, gout, gom, reach, codes, boxes, stream)
                   : launch_samples_typed<T, VEC, 3, 3, false>(g, value, om, gout, gom, reach, codes, boxes, stream);
    }
    return launch_samples_typed<T, VEC, 0, 0, false>(g, value, om, gout, gom, reach, codes, boxes, stream);
}

template <typename T>
cudaError_t launch_samples_vec(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                               int* reach, void* codes, uint32_t* boxes, cudaStream_t stream) {
    return g.vec == 2 ? launch_samples_grid<T, 2>(g, value, om, gout, gom, reach, codes, boxes, stream)
                      : launch_samples_grid<T, 1>(g, value, om, gout, gom, reach, codes, boxes, stream);
}

template <typename T, int VEC>
cudaError_t launch_value_typed(const Geometry& g, const void* om, const void* gout, void* gvalue, const int* reach,
                               const void* codes, const uint32_t* boxes, cudaStream_t stream) {
    const size_t smem = backward_value_smem_bytes(g);
    auto kern = value_kernel<T, VEC, sizeof(T) == 2>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const long long blocks = static_cast<long long>(g.N) * g.btiles_h * g.btiles_w;
    kern<<<static_cast<unsigned>(blocks), g.bthreads, smem, stream>>>(
        g, static_cast<const T*>(om), static_cast<const T*>(gout), static_cast<T*>(gvalue), reach, codes, boxes);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_value_vec(const Geometry& g, const void* om, const void* gout, void* gvalue, const int* reach,
                             const void* codes, const uint32_t* boxes, cudaStream_t stream) {
    return g.vec == 2 ? launch_value_typed<T, 2>(g, om, gout, gvalue, reach, codes, boxes, stream)
                      : launch_value_typed<T, 1>(g, om, gout, gvalue, reach, codes, boxes, stream);
}

}  // namespace

size_t backward_smem_bytes(const Geometry& g, int elem_bytes) {
    return static_cast<size_t>(g.TH) * g.TW * g.P * elem_bytes * 2;
}

size_t backward_value_smem_bytes(const Geometry& g) {
    const size_t nbins = static_cast<size_t>(g.G) * (g.BH + 1) * (g.BW + 1);
    return ((2 * nbins + kListCap) * sizeof(int) + 15) / 16 * 16 + static_cast<size_t>(g.bcap) * g.brec;
}

cudaError_t launch_backward_samples(const Geometry& g, int dtype, const void* value, const void* om, const void* gout,
                                    void* gom, int* reach, void* codes, uint32_t* boxes, cudaStream_t stream) {
    switch (dtype) {
        case 0: return launch_samples_vec<float>(g, value, om, gout, gom, reach, codes, boxes, stream);
        case 1: return launch_samples_vec<__half>(g, value, om, gout, gom, reach, codes, boxes, stream);
        case 2: return launch_samples_vec<__nv_bfloat16>(g, value, om, gout, gom, reach, codes, boxes, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_backward_value(const Geometry& g, int dtype, const void* om, const void* gout, void* gvalue,
                                  const int* reach, const void* codes, const uint32_t* boxes,
                                  cudaStream_t stream) {
    switch (dtype) {
        case 0: return launch_value_vec<float>(g, om, gout, gvalue, reach, codes, boxes, stream);
        case 1: return launch_value_vec<__half>(g, om, gout, gvalue, reach, codes, boxes, stream);
        case 2: return launch_value_vec<__nv_bfloat16>(g, om, gout, gvalue, reach, codes, boxes, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
