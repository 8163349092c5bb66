// dcn4_backward.cu — gradients of the DCNv4 core spatial aggregation.
//
// For every sample (output pixel p, group g, point k) with location
// (h, w) = anchor + s*(dy, dx), bilinear cell corners v_ab and weights
// w_ab = (a ? lh : 1-lh)(b ? lw : 1-lw), and gy = grad_out of (p, g):
//   d/d m_k   = <gy, S>,                        S = sum_ab w_ab v_ab
//   d/d dx_k  = s * m_k * <gy, dS/dw>,          dS/dw = (1-lh)(v01 - v00) + lh(v11 - v10)
//   d/d dy_k  = s * m_k * <gy, dS/dh>,          dS/dh = (1-lw)(v10 - v00) + lw(v11 - v01)
//   grad_value[corner ab] += m_k * w_ab * gy     (every in-image corner)
// where <.,.> sums over the group's C' channels.  With g.softmax the masks
// are logits l_k and m_k = softmax(l)_k over the K points of the (pixel,
// group) (the DCNv3 form); m_k then stands for that weight above, and
//   d/d l_k   = m_k * (<gy, S_k> - sum_j m_j <gy, S_j>)
// (the softmax Jacobian applied to the gradients of the weights).
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
//   touches the image; per output pixel, the bounding box of its samples'
//   cells; and, per sample, a 2-byte code of its cell relative to its anchor
//   (for 16-bit dtypes also the mask bits and fixed-point lh, lw).
//
// value_kernel (input tiles).  grad_value is pulled, not scattered: a CTA owns
//   a BH x BW tile of input pixels (all groups) and writes each of their
//   grad_value elements exactly once.  The samples that can touch the tile come
//   from output pixels whose anchors lie within R of it and whose cell box
//   meets the tile; the CTA reads those samples' cell codes and counting-sorts
//   the ones whose cell touches the tile by (group, cell) in shared memory.
//   Then lanes own cell columns and walk cell rows: each sample is read once
//   and added to its cell's four corners, and a shuffle joins the corners a
//   pixel shares with the next column.  Should the sorted samples not fit in
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

// Per-sample entries the sample pass leaves for the grad_value pass.  fp32
// I/O: the 2-byte cell code only (the grad_value pass re-forms the exact
// weights from the offsets).  16-bit I/O: also the mask's own 16 bits and lh,
// lw as 16-bit fixed point, so the grad_value pass never reads the offsets.
// The three live in separate arrays: the scan that filters candidates reads
// only the codes.

__device__ __forceinline__ uint32_t fix16(float f) { return min(65535u, static_cast<uint32_t>(f * 65536.f + 0.5f)); }

// A softmax weight (in [0, 1]) in the 16 mask bits of a compact record: q / 65535
// (absolute error below 2^-17, like the bilinear fractions).
__device__ __forceinline__ uint32_t weight_q16(float a) { return min(65535u, static_cast<uint32_t>(a * 65535.f + 0.5f)); }
constexpr float kWeightQ16 = 0x1p-32f / 65535.f;  // q16 weight x 2^-32 (the fractions' scale) per unit of q

template <typename T>
__device__ __forceinline__ uint16_t raw_bits(T x) {
    uint16_t b;
    memcpy(&b, &x, 2);
    return b;
}

// An fp32 value in the two elements at p (one element for fp32 storage), as
// raw bits; get_f32 reads it back.
__device__ __forceinline__ void put_f32(float* p, float v) { *p = v; }
__device__ __forceinline__ float get_f32(const float* p) { return *p; }
__device__ __forceinline__ void put_f32(__half* p, float v) {
    const uint32_t b = __float_as_uint(v);
    p[0] = __ushort_as_half(static_cast<unsigned short>(b & 0xffffu));
    p[1] = __ushort_as_half(static_cast<unsigned short>(b >> 16));
}
__device__ __forceinline__ float get_f32(const __half* p) {
    return __uint_as_float(static_cast<uint32_t>(__half_as_ushort(p[0])) | (static_cast<uint32_t>(__half_as_ushort(p[1])) << 16));
}
__device__ __forceinline__ void put_f32(__nv_bfloat16* p, float v) {
    const uint32_t b = __float_as_uint(v);
    p[0] = __ushort_as_bfloat16(static_cast<unsigned short>(b & 0xffffu));
    p[1] = __ushort_as_bfloat16(static_cast<unsigned short>(b >> 16));
}
__device__ __forceinline__ float get_f32(const __nv_bfloat16* p) {
    return __uint_as_float(static_cast<uint32_t>(__bfloat16_as_ushort(p[0])) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(p[1])) << 16));
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
// Filing (16-bit dtypes, when g.buckets): the grad_offset_mask CTA files each
// sample under every grad_value tile whose cells hold it -- the tile holding
// the cell's top-left pixel (h0, w0) (tile row 0 for h0 = -1, likewise for
// columns), and the next tile down / right as well when the cell straddles
// that boundary.  Records are staged in shared memory with their rank among
// the CTA's records for the same tile; after the samples the CTA takes one
// range per tile from the tile's global counter and writes its records there
// (records of one tile keep no particular order).  Tiles are named by their
// place in a window of kFileSlots tiles around the CTA's anchors (g.fwin_h
// tile rows x 2^g.fwin_wl tile columns: square for tall tiles, tall and
// narrow when grad_value tiles are only a row or two high); a
// record for a tile outside the window, or beyond the staging room, marks the
// tile kBucketOverflow instead, and that tile rescans the offsets.
// ---------------------------------------------------------------------------
constexpr int kFileSlots = 64;

// Staging of one (sample, thread): the record for the cell's own tile (bin
// included) and a meta word: window slot of that tile (6 bits), the record's
// rank there and the ranks of its copies for the tile below, right and
// below-right (13 bits each), a flag per copy (bits 58-60), and bit 61 when
// the own-tile record exists.  A copy's bin follows from the cell's: a cell
// on the bottom border (cell row BH) is cell row 0 below, one on the right
// border (cell column BW) is cell column 0 to the right.
struct FileStage {
    uint64_t* rec;   // [K][threads]
    uint64_t* meta;  // [K][threads]
    int wy0, wx0;    // window origin (tile row, tile column)
    int wh, wwl;     // window rows, log2 of its columns (wh << wwl == kFileSlots)
};
constexpr int kRankBits = 13;  // ranks < K * threads <= 2^13 (checked on the host)

__device__ __forceinline__ int window_slot(const FileStage& fs, int ty, int tx) {
    const int dy = ty - fs.wy0, dx = tx - fs.wx0;
    return (static_cast<unsigned>(dy) < static_cast<unsigned>(fs.wh) &&
            static_cast<unsigned>(dx) < static_cast<unsigned>(1 << fs.wwl))
               ? (dy << fs.wwl) + dx
               : -1;
}

__device__ __forceinline__ int tile_index(const Geometry& g, int n, int ty, int tx) {
    return (n * g.btiles_h + ty) * g.btiles_w + tx;
}

// ---------------------------------------------------------------------------
// grad_offset_mask + reach
// ---------------------------------------------------------------------------
template <typename T, int VEC, int KH, int KW, bool RC, bool SM>
__global__ void __launch_bounds__(256, 3) samples_kernel(const Geometry g, const T* __restrict__ value,
                                                      const T* __restrict__ om, const T* __restrict__ gout,
                                                      T* __restrict__ gom, int* __restrict__ reach,
                                                      const SampleArrays sa, uint32_t* __restrict__ boxes) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_reach;
    __shared__ int s_box[4 * 256];  // per tile pixel: min/max cell row, min/max cell column (relative)
    __shared__ int s_fcnt[kFileSlots], s_fbase[kFileSlots];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    const int tile_elems = g.TH * g.TW * g.P;
    T* om_s = reinterpret_cast<T*>(smem);
    T* gom_s = reinterpret_cast<T*>(smem + tile_elems * sizeof(T));  // P % 8 == 0 keeps this 16-byte aligned
    const bool filing = sizeof(T) == 2 && g.buckets != 0;
    // Unrolled grids without softmax or remove_center stage only the meta words:
    // the record body (bin, mask bits, fractions) is formed again at write-out
    // from the offsets, which stay in shared memory, with the same fp32
    // arithmetic.  Half the staging leaves that much more of the SM's L1 to the
    // gathers (measured: a gain where the samples spread wide, a small loss
    // with remove_center at every offset scale tried).
    constexpr bool SLIM = KH > 0 && !SM && !RC;

    const Tile t = tile_of_block(g);
    const int K = KH > 0 ? KH * KW - (RC ? 1 : 0) : g.K;
    const int kh = KH > 0 ? KH : g.kh;
    const int kw = KW > 0 ? KW : g.kw;
    const bool rc = KH > 0 ? RC : g.remove_center != 0;
    FileStage fs;
    if (filing) {
        // staging after the two offset_mask tiles
        unsigned char* st = smem + 2 * static_cast<size_t>(tile_elems) * sizeof(T);
        fs.rec = reinterpret_cast<uint64_t*>(st);
        fs.meta = SLIM ? fs.rec : fs.rec + (KH > 0 ? K : filing_chunk(g)) * blockDim.x;
        // window of tiles centred on the anchors of this CTA's grid
        const int amid_h = t.ho0 * g.sh - g.ph + ((t.th - 1) * g.sh + (kh - 1) * g.dh) / 2;
        const int amid_w = t.wo0 * g.sw - g.pw + ((t.tw - 1) * g.sw + (kw - 1) * g.dw) / 2;
        fs.wh = KH > 0 ? 8 : g.fwin_h;  // the unrolled grids are compiled for an 8 x 8 window
        fs.wwl = KH > 0 ? 3 : g.fwin_wl;
        fs.wy0 = max(0, max(0, amid_h) / g.BH - fs.wh / 2);
        fs.wx0 = max(0, max(0, amid_w) / g.BW - (1 << fs.wwl) / 2);
        for (int i = threadIdx.x; i < kFileSlots; i += blockDim.x) s_fcnt[i] = 0;
    }
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
    const int lrow = (active ? lp : 0) * g.P + grp * 3 * K;
    const T* row = om_s + lrow;
    const int ch_off = grp * g.Cg + sl * (VEC * EPV);
    const T* img = value + static_cast<long long>(t.n) * g.H * g.W * g.C + ch_off;
    const int hb = ho * g.sh - g.ph, wb = wo * g.sw - g.pw;

    float2 gy[PAIRS];
    const long long pix = (static_cast<long long>(t.n) * g.Ho + ho) * g.Wo + wo;
    load_gy<T, VEC>(gy, gout + pix * g.C + ch_off);
    const long long s0 = (pix * g.G + grp) * K;  // first entry of this (pixel, group): [N, Ho, Wo, G, K]
    const bool writer = active && sl == 0;
    int my_reach = -1;
    int bmin_h = 127, bmax_h = -128, bmin_w = 127, bmax_w = -128;  // cells relative to (hb, wb)
    constexpr bool smax = SM;  // masks are logits (softmax over the K points)
    float2 stats = make_float2(0.f, 1.f);  // softmax: (l_max, 1 / sum_k exp(l_k - l_max))
    if constexpr (SM) stats = softmax_stats(row + 2 * K, K);
    float gdot = 0.f;  // softmax: sum_k m_k <gy, S_k>

    // Filing write-out: one range per window tile from its global counter, then
    // the nk staged points of each thread.
    auto reserve = [&]() {
        const int wmask = (1 << fs.wwl) - 1;
        for (int i = threadIdx.x; i < kFileSlots; i += blockDim.x) {
            s_fbase[i] = 0;
            if (s_fcnt[i] > 0)
                s_fbase[i] = atomicAdd(sa.tile_count + tile_index(g, t.n, fs.wy0 + (i >> fs.wwl), fs.wx0 + (i & wmask)),
                                       s_fcnt[i]);
        }
    };
    auto write_out = [&](int nk) {
        const int wmask = (1 << fs.wwl) - 1;
        const uint32_t pixv = (static_cast<uint32_t>(t.ho0 + (active ? py : 0)) << 16) |
                              static_cast<uint32_t>(t.wo0 + (active ? px : 0));
        auto put = [&](int dl, int rank, uint64_t rec) {
            const int slot = s_fbase[dl] + rank;
            if (static_cast<unsigned>(slot) >= static_cast<unsigned>(g.bcap)) return;  // the tile rescans
            const long long at = static_cast<long long>(tile_index(g, t.n, fs.wy0 + (dl >> fs.wwl), fs.wx0 + (dl & wmask))) *
                                     g.bcap + slot;
            sa.bucket_pix[at] = pixv;
            sa.bucket_rec[at] = rec;
        };
        const int rmask = (1 << kRankBits) - 1;
        auto emit = [&](uint64_t meta, uint64_t rec) {
            const int dl0 = static_cast<int>(meta & 63);
            put(dl0, static_cast<int>(meta >> 6) & rmask, rec);
            const uint64_t body = rec & ~0xffffull;
            const int bin = static_cast<int>(rec & 0xffff);
            if ((meta >> 58) & 1)  // below: cell row 0 there
                put(dl0 + (1 << fs.wwl), static_cast<int>(meta >> (6 + kRankBits)) & rmask,
                    body | static_cast<uint64_t>(bin - g.BH * (g.BW + 1)));
            if ((meta >> 59) & 1)  // right: cell column 0 there
                put(dl0 + 1, static_cast<int>(meta >> (6 + 2 * kRankBits)) & rmask, body | static_cast<uint64_t>(bin - g.BW));
            if ((meta >> 60) & 1)  // below-right
                put(dl0 + (1 << fs.wwl) + 1, static_cast<int>(meta >> (6 + 3 * kRankBits)) & rmask,
                    body | static_cast<uint64_t>(bin - g.BH * (g.BW + 1) - g.BW));
        };
        if constexpr (SLIM) {
            // Walk the grid as the sample loop did, so the anchors are compile-time
            // offsets; the cell's tile comes back from the staged window slot.
            const int gbase = grp * (g.BH + 1) * (g.BW + 1);
            int j = 0;
#pragma unroll
            for (int iw = 0; iw < KW; ++iw) {
#pragma unroll
                for (int ih = 0; ih < KH; ++ih) {
                    if (RC && iw == KW / 2 && ih == KH / 2) continue;
                    const int kk = j++;
                    const uint64_t meta = fs.meta[kk * blockDim.x + threadIdx.x];
                    if (!((meta >> 61) & 1)) continue;
                    const int dl0 = static_cast<int>(meta & 63);
                    const int ta = fs.wy0 + (dl0 >> fs.wwl), ua = fs.wx0 + (dl0 & wmask);
                    const float h = __fmaf_rn(g.s, to_f32(row[2 * kk + 1]), static_cast<float>(hb + ih * g.dh));
                    const float w = __fmaf_rn(g.s, to_f32(row[2 * kk]), static_cast<float>(wb + iw * g.dw));
                    const float h0f = floorf(h), w0f = floorf(w);
                    const int cy = static_cast<int>(h0f) + 1 - ta * g.BH, cx = static_cast<int>(w0f) + 1 - ua * g.BW;
                    const uint64_t rec = (static_cast<uint64_t>(raw_bits(row[2 * K + kk])) << 16) |
                                         (static_cast<uint64_t>(fix16(h - h0f)) << 32) |
                                         (static_cast<uint64_t>(fix16(w - w0f)) << 48) |
                                         static_cast<uint64_t>(gbase + cy * (g.BW + 1) + cx);
                    emit(meta, rec);
                }
            }
        } else {
            for (int j = 0; j < nk; ++j) {
                const int at = j * blockDim.x + threadIdx.x;
                const uint64_t meta = fs.meta[at];
                if (!((meta >> 61) & 1)) continue;
                emit(meta, fs.rec[at]);
            }
        }
    };
    // Generic grids file in chunks of filing_chunk(g) points (a bounded staging area).
    const int fkc = KH > 0 ? K : filing_chunk(g);
    int kc = 0;  // points staged in the current chunk

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
            float m = to_f32(row[2 * K + kk]);
            if constexpr (SM) m = softmax_weight(m, stats);
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
            float gw = 0.f;  // <gy, S_k>
            if (cell.any) {
                if (sl == 0) {
                    const float hl = 1.f - cell.lh, wl = 1.f - cell.lw;
                    const float sm = g.s * m;
                    T* gr = gom_s + lrow;  // rounded once, to the I/O dtype
                    gr[2 * kk] = from_f32<T>(sm * (hl * (d01 - d00) + cell.lh * (d11 - d10)));
                    gr[2 * kk + 1] = from_f32<T>(sm * (wl * (d10 - d00) + cell.lw * (d11 - d01)));
                    gw = hl * (wl * d00 + cell.lw * d01) + cell.lh * (wl * d10 + cell.lw * d11);
                    if (!smax) gr[2 * K + kk] = from_f32<T>(gw);
                }
                const int dh = max(abs(cell.h0 - ah), abs(cell.h0 + 1 - ah));
                const int dw = max(abs(cell.w0 - aw), abs(cell.w0 + 1 - aw));
                my_reach = max(my_reach, max(dh, dw));
                bmin_h = min(bmin_h, cell.h0 - hb);
                bmax_h = max(bmax_h, cell.h0 - hb);
                bmin_w = min(bmin_w, cell.w0 - wb);
                bmax_w = max(bmax_w, cell.w0 - wb);
            }
            if (smax && writer) {
                // the staged offsets of sample kk are spent: they keep <gy, S_k> (fp32 bits)
                put_f32(om_s + lrow + 2 * kk, gw);
                gdot = __fmaf_rn(m, gw, gdot);
            }
            if constexpr (sizeof(T) == 2) {
                if (filing) {
                    const bool has = writer && cell.any;
                    const int h0 = cell.h0, w0 = cell.w0;
                    const int ta = h0 < 0 ? 0 : g.BH == 1 ? h0 : static_cast<int>(__umulhi(static_cast<uint32_t>(h0), g.bh_magic));
                    const int ua = w0 < 0 ? 0 : g.BW == 1 ? w0 : static_cast<int>(__umulhi(static_cast<uint32_t>(w0), g.bw_magic));
                    const int cy = h0 + 1 - ta * g.BH, cx = w0 + 1 - ua * g.BW;
                    const int gbase = grp * (g.BH + 1) * (g.BW + 1);
                    const uint64_t mbits = smax ? weight_q16(m) : raw_bits(row[2 * K + kk]);
                    const uint64_t rec = (mbits << 16) |
                                         (static_cast<uint64_t>(fix16(cell.lh)) << 32) |
                                         (static_cast<uint64_t>(fix16(cell.lw)) << 48);
                    const int dl0 = has ? window_slot(fs, ta, ua) : -1;
                    if (has && dl0 < 0) {
                        // The own tile is outside the window: it rescans, and so do the tiles this
                        // sample's copies would have gone to, since none of them gets its record.
                        atomicOr(sa.tile_count + tile_index(g, t.n, ta, ua), kBucketOverflow);
                        const bool sr = h0 >= 0 && h0 + 1 < g.H && h0 + 1 == (ta + 1) * g.BH;
                        const bool sc = w0 >= 0 && w0 + 1 < g.W && w0 + 1 == (ua + 1) * g.BW;
                        if (sr) atomicOr(sa.tile_count + tile_index(g, t.n, ta + 1, ua), kBucketOverflow);
                        if (sc) atomicOr(sa.tile_count + tile_index(g, t.n, ta, ua + 1), kBucketOverflow);
                        if (sr && sc) atomicOr(sa.tile_count + tile_index(g, t.n, ta + 1, ua + 1), kBucketOverflow);
                    }
                    // rank among the CTA's records for the tile: one shared atomic per distinct tile in the warp
                    const unsigned okm = __ballot_sync(0xffffffffu, dl0 >= 0);
                    uint64_t meta = 0;
                    if (dl0 >= 0) {
                        const int lane = threadIdx.x & 31;
                        const unsigned peers = __match_any_sync(okm, dl0);
                        const int leader = __ffs(peers) - 1;
                        int base = 0;
                        if (lane == leader) base = atomicAdd(s_fcnt + dl0, __popc(peers));
                        // every lane with a record takes part (one mask for all), each reading its own leader
                        base = __shfl_sync(okm, base, leader);
                        const int rank = base + __popc(peers & ((1u << lane) - 1));
                        meta = static_cast<uint64_t>(dl0) | (static_cast<uint64_t>(rank) << 6) | (1ull << 61);
                        // copies for the next tiles when the cell straddles a border
                        const bool dup_r = h0 >= 0 && h0 + 1 < g.H && h0 + 1 == (ta + 1) * g.BH;
                        const bool dup_c = w0 >= 0 && w0 + 1 < g.W && w0 + 1 == (ua + 1) * g.BW;
#pragma unroll
                        for (int d = 1; d < 4; ++d) {
                            if (!((d == 1 && dup_r) || (d == 2 && dup_c) || (d == 3 && dup_r && dup_c))) continue;
                            const int ty = ta + (d & 1), tx = ua + (d >> 1);
                            const int dl = window_slot(fs, ty, tx);
                            if (dl < 0) {
                                atomicOr(sa.tile_count + tile_index(g, t.n, ty, tx), kBucketOverflow);
                                continue;
                            }
                            const int r = atomicAdd(s_fcnt + dl, 1);
                            meta |= (static_cast<uint64_t>(r) << (6 + kRankBits * d)) | (1ull << (57 + d));
                        }
                    }
                    const int at = (KH > 0 ? kk : kc) * blockDim.x + threadIdx.x;
                    fs.meta[at] = meta;
                    if constexpr (!SLIM) fs.rec[at] = rec | static_cast<uint64_t>(gbase + cy * (g.BW + 1) + cx);
                    if constexpr (KH == 0) {
                        // every thread takes the same branch: kc, kk and filing are uniform
                        if (++kc == fkc || kk + 1 == K) {
                            __syncthreads();
                            reserve();
                            __syncthreads();
                            write_out(kc);
                            __syncthreads();
                            for (int i = threadIdx.x; i < kFileSlots; i += blockDim.x) s_fcnt[i] = 0;
                            __syncthreads();
                            kc = 0;
                        }
                    }
                }
            } else {
                if (writer) sa.code[s0 + kk] = cell_code(cell.any, cell.h0 - ah, cell.w0 - aw);
            }
        }
    }

    if (smax && writer) {
        // logit gradients: the softmax Jacobian applied to the weight gradients
        T* gr = gom_s + lrow;
        for (int kk = 0; kk < K; ++kk)
            gr[2 * K + kk] = from_f32<T>(softmax_weight(to_f32(row[2 * K + kk]), stats) * (get_f32(row + 2 * kk) - gdot));
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
    if (KH > 0 && filing) {  // the unrolled grids stage all K points and file them here
        reserve();
        __syncthreads();
        write_out(K);
    }
    if (threadIdx.x == 0 && s_reach >= 0) atomicMax(reach + t.n, s_reach + 1);  // stored as R + 1; 0: no sample
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

// Sample records of the grad_value sort.  Wide (16 bytes, fp32 I/O): grad_out
// offset of the sample's output pixel p, m(1-lh), m lh, lw.  Compact (8 bytes,
// 16-bit I/O): p relative to the tile's reference output pixel (ho_ref - 64,
// wo_ref - 64) as 7 + 7 bits, the mask's own 16 bits, and lh, lw as 16-bit
// fixed point (error below 2^-17, far under the I/O rounding).
__device__ __forceinline__ float from_bits(uint16_t b, __half) {
    __half h;
    memcpy(&h, &b, 2);
    return __half2float(h);
}
__device__ __forceinline__ float from_bits(uint16_t b, __nv_bfloat16) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Where a record's grad_out slice is: compact records add their 7-bit row and
// column to `ref` (row stride `row`, column stride `col`, in elements); wide
// records carry the offset from `ref` themselves.
template <typename T>
struct GySource {
    const T* ref;
    int row, col;
};

// Adds U consecutive sorted records (from index j) of one cell to the partial
// sums of its four corners: t0/t1 = top-left/top-right, b0/b1 = bottom-left/
// bottom-right.  All U grad_out gathers are issued before any is used.
template <typename T, int VEC, bool COMPACT, int U>
__device__ __forceinline__ void pull_records(const unsigned char* rec_base, const GySource<T>& gs, bool smax, int j,
                                             float2* t0, float2* t1, float2* b0, float2* b1) {
    constexpr int EPV = Elem<T>::per16;
    const T* src[U];
    float w[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if constexpr (COMPACT) {
            const uint2 r = reinterpret_cast<const uint2*>(rec_base)[j + u];
            // m * (hq * wq) * 2^-32 with hq, wq the 16-bit fixed-point weights; m is
            // the mask's own bits, or with softmax its weight as q / 65535
            const uint32_t mq = r.x >> 16;
            const float ms = smax ? static_cast<float>(mq) * kWeightQ16 : from_bits(static_cast<uint16_t>(mq), T()) * 0x1p-32f;
            const float hq1 = static_cast<float>(r.y & 0xffff), hq0 = 65536.f - hq1;
            const float wq1 = static_cast<float>(r.y >> 16), wq0 = 65536.f - wq1;
            w[u][0] = ms * (hq0 * wq0);
            w[u][1] = ms * (hq0 * wq1);
            w[u][2] = ms * (hq1 * wq0);
            w[u][3] = ms * (hq1 * wq1);
            src[u] = gs.ref + static_cast<int>(r.x & 127) * gs.row + static_cast<int>((r.x >> 7) & 127) * gs.col;
        } else {
            const float4 r = reinterpret_cast<const float4*>(rec_base)[j + u];
            const float lw0 = 1.f - r.w;
            w[u][0] = r.y * lw0;
            w[u][1] = r.y * r.w;
            w[u][2] = r.z * lw0;
            w[u][3] = r.z * r.w;
            src[u] = gs.ref + __float_as_int(r.x);
        }
    }
    uint4 raw[U][VEC];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if constexpr (VEC == 2) {
            ld_keep32(src[u], raw[u][0], raw[u][1]);
        } else {
            raw[u][0] = ld_keep16(src[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const float2 w00 = make_float2(w[u][0], w[u][0]), w01 = make_float2(w[u][1], w[u][1]);
        const float2 w10 = make_float2(w[u][2], w[u][2]), w11 = make_float2(w[u][3], w[u][3]);
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            float2 f[EPV / 2];
            unpack(raw[u][v], f, T());
#pragma unroll
            for (int i = 0; i < EPV / 2; ++i) {
                const int k = v * (EPV / 2) + i;
                t0[k] = __ffma2_rn(w00, f[i], t0[k]);
                t1[k] = __ffma2_rn(w01, f[i], t1[k]);
                b0[k] = __ffma2_rn(w10, f[i], b0[k]);
                b1[k] = __ffma2_rn(w11, f[i], b1[k]);
            }
        }
    }
}

// All records [j, end) of one cell, two at a time.
template <typename T, int VEC, bool COMPACT>
__device__ __forceinline__ void pull_cell(const unsigned char* rec_base, const GySource<T>& gs, bool smax, int j,
                                          int end, float2* t0, float2* t1, float2* b0, float2* b1) {
    for (; j + 1 < end; j += 2) pull_records<T, VEC, COMPACT, 2>(rec_base, gs, smax, j, t0, t1, b0, b1);
    if (j < end) pull_records<T, VEC, COMPACT, 1>(rec_base, gs, smax, j, t0, t1, b0, b1);
}

// A finished pixel row of a strip: lane cx holds the right corners (r) of
// pixel cx and the left corners (l) of pixel cx - 1; the pixel's sum is its
// own r plus the next lane's l.  Stores it (when `store`) and clears l, r.
template <typename T, int VEC>
__device__ __forceinline__ void finish_row(float2* l, float2* r, int LW, bool store, T* dst) {
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    float2 out[PAIRS];
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) {
        out[i].x = r[i].x + __shfl_down_sync(0xffffffffu, l[i].x, 1, LW);
        out[i].y = r[i].y + __shfl_down_sync(0xffffffffu, l[i].y, 1, LW);
    }
    if (store) {
        if constexpr (VEC == 2) {
            st_global32(dst, pack(out, T()), pack(out + EPV / 2, T()));
        } else {
            st_global(dst, pack(out, T()));
        }
    }
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) l[i] = r[i] = make_float2(0.f, 0.f);
}

// Exclusive scan of cnt[0, nbins) into cur, block-wide (thread-contiguous
// chunks); every thread gets the total.  Starts and ends with a barrier.
__device__ __forceinline__ int bins_exclusive_scan(const int* cnt, int* cur, int nbins, int* s_warp, int* s_total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    __syncthreads();
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
        if (lane == nwarps - 1) *s_total = v;
    }
    __syncthreads();
    int run = incl - local + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int b = b0; b < min(nbins, b0 + per); ++b) {
        cur[b] = run;
        run += cnt[b];
    }
    __syncthreads();
    return *s_total;
}

// Compact record of a sample of output pixel (ho, wo): false if the pixel is
// outside the 128 x 128 window the record can name.
__device__ __forceinline__ bool compact_source(int ho, int wo, int ho_ref, int wo_ref, uint32_t& id) {
    const int dh = ho - ho_ref + 64, dw = wo - wo_ref + 64;
    id = static_cast<uint32_t>(dh) | (static_cast<uint32_t>(dw) << 7);
    return static_cast<unsigned>(dh) < 128u && static_cast<unsigned>(dw) < 128u;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    unsigned r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Records of the grad_value sort each thread keeps in flight.
constexpr int kScanBatch = 8;

template <typename T, int VEC, bool COMPACT, bool SM>
__global__ void __launch_bounds__(256, 2) value_kernel(const Geometry g, const T* __restrict__ om,
                                                       const T* __restrict__ gout, T* __restrict__ gvalue,
                                                       const int* __restrict__ reach, const SampleArrays sa,
                                                       const uint32_t* __restrict__ boxes) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_warp[32];
    __shared__ int s_total;
    __shared__ int s_nlist;
    __shared__ int s_fail;
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;

    // Input tile of this CTA.
    const int per_img = g.btiles_h * g.btiles_w;
    const int n = blockIdx.x / per_img;
    const int tr = blockIdx.x - n * per_img;
    const int by = tr / g.btiles_w;
    const int y0 = by * g.BH, x0 = (tr - by * g.btiles_w) * g.BW;
    const int bh = min(g.BH, g.H - y0), bw = min(g.BW, g.W - x0);
    // Cell (bin) (cy, cx) of the tile has its top-left corner at pixel
    // (y0 - 1 + cy, x0 - 1 + cx); cy in [0, bh], cx in [0, bw].
    const int cells_w = g.BW + 1;
    const int cells = (g.BH + 1) * cells_w;
    const int nbins = g.G * cells;
    const int GK = g.G * g.K;
    int* cnt = reinterpret_cast<int*>(smem);
    int* cur = cnt + nbins;
    uint32_t* s_list = reinterpret_cast<uint32_t*>(cur + nbins);  // candidate pixels: (ho << 16) | wo
    int4* s_tab = reinterpret_cast<int4*>(smem + ((2 * nbins + kListCap) * sizeof(int) + 15) / 16 * 16);
    unsigned char* rec_base = reinterpret_cast<unsigned char*>(s_tab + GK);
    float4* rec_w = reinterpret_cast<float4*>(rec_base);
    uint2* rec_c = reinterpret_cast<uint2*>(rec_base);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int nthr = blockDim.x;
    const long long pix0 = static_cast<long long>(n) * g.Ho * g.Wo;
    constexpr bool smax = SM;  // weights are the softmax of each (pixel, group)'s logits
    // Compact records name their output pixel relative to this one (a sample
    // of output pixel p touches the tile only if p's grid lies near it).
    const int ho_ref = floor_div(y0 + g.ph, g.sh), wo_ref = floor_div(x0 + g.pw, g.sw);
    // ... and the pull forms their grad_out offsets in 32 bits.
    const bool compact_ok = !COMPACT || 128LL * (g.Wo + 1) * g.C < (1LL << 31);

    if (threadIdx.x == 0) {
        s_nlist = 0;
        s_fail = 0;
    }
    for (int i = threadIdx.x; i < nbins; i += nthr) cnt[i] = 0;

    bool sorted = false;
    const int R = reach[n] - 1;  // -1: no sample of the image touches it
    // The filing pass trusts the cell codes only up to kCodeReach.
    const int nfiled = (COMPACT && g.buckets && compact_ok && R <= kCodeReach) ? sa.tile_count[blockIdx.x] : -1;
    if (nfiled >= 0 && nfiled <= g.bcap) {
        // The grad_offset_mask pass filed this tile's records in its bucket:
        // count them per bin, scan, place them in bin order.
        const uint64_t* brec = sa.bucket_rec + static_cast<long long>(blockIdx.x) * g.bcap;
        const uint32_t* bpix = sa.bucket_pix + static_cast<long long>(blockIdx.x) * g.bcap;
        __syncthreads();
        for (int i0 = threadIdx.x; i0 < nfiled; i0 += kScanBatch * nthr) {
            uint32_t bin[kScanBatch];
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u) {
                const int i = i0 + u * nthr;
                bin[u] = i < nfiled ? ld_stream_u16(brec + i) : 0xffffffffu;
            }
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u) {
                if (bin[u] == 0xffffffffu) continue;
                // A bin outside the tile means a corrupt bucket: never index with it; the
                // tile then takes the direct path.
                if (bin[u] >= static_cast<uint32_t>(nbins)) {
                    s_fail = 1;
                    continue;
                }
                atomicAdd(&cnt[bin[u]], 1);
            }
        }
        bins_exclusive_scan(cnt, cur, nbins, s_warp, &s_total);
        for (int i0 = threadIdx.x; i0 < nfiled; i0 += kScanBatch * nthr) {
            uint64_t r[kScanBatch];
            uint32_t p[kScanBatch];
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u) {
                const int i = i0 + u * nthr;
                r[u] = 0;
                p[u] = 0;
                if (i < nfiled) {
                    r[u] = ld_stream_u64(brec + i);
                    p[u] = ld_stream_u32(bpix + i);
                }
            }
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u) {
                if (i0 + u * nthr >= nfiled) continue;
                uint32_t id;
                const uint32_t bin = static_cast<uint32_t>(r[u]) & 0xffff;
                if (bin >= static_cast<uint32_t>(nbins) ||
                    !compact_source(static_cast<int>(p[u] >> 16), static_cast<int>(p[u] & 0xffff), ho_ref, wo_ref, id)) {
                    s_fail = 1;
                    continue;
                }
                const int slot = atomicAdd(&cur[bin], 1);
                if (slot >= nfiled) {  // more records of a bin than counted: corrupt bucket
                    s_fail = 1;
                    continue;
                }
                rec_c[slot] = make_uint2(id | (static_cast<uint32_t>(r[u]) & 0xffff0000u), static_cast<uint32_t>(r[u] >> 32));
            }
        }
        __syncthreads();
        sorted = s_fail == 0;
        // A bucket that failed the checks: counted, so that callers and tests can
        // tell that it happened (the tile's result is still exact).
        if (!sorted && threadIdx.x == 0) atomicAdd(sa.diag + kDiagCorruptBucket, 1);
    } else {
        if (COMPACT && g.buckets && threadIdx.x == 0) atomicAdd(sa.diag + kDiagRescan, 1);
        // Rescan: samples that can touch the tile come from output pixels
        // whose anchor (for the sample's grid point) lies within R of the tile
        // and whose cell box meets the tile's cells.
        for (int gk = threadIdx.x; gk < GK; gk += nthr) {
            // Per (group, point): bin offset of the group, and the anchor of the
            // point relative to the tile's first cell (anchor row = ho*sh + .y,
            // column = wo*sw + .z); .w = point | group << 16.
            const int sg = gk / g.K, sk = gk - (gk / g.K) * g.K;
            int ih, iw;
            grid_cell_of(g, sk, ih, iw);
            s_tab[gk] = make_int4(sg * cells, ih * g.dh - g.ph - (y0 - 1), iw * g.dw - g.pw - (x0 - 1), sk | (sg << 16));
        }
        const bool boxes_exact = R <= kCodeReach && R + max((g.kh - 1) * g.dh, (g.kw - 1) * g.dw) <= 127;
        int ho_lo = 0, ho_hi = -1, wo_lo = 0, wo_hi = -1;
        if (R >= 0) {
            ho_lo = max(0, ceil_div(y0 - R + g.ph - (g.kh - 1) * g.dh, g.sh));
            ho_hi = min(g.Ho - 1, floor_div(y0 + bh - 1 + R + g.ph, g.sh));
            wo_lo = max(0, ceil_div(x0 - R + g.pw - (g.kw - 1) * g.dw, g.sw));
            wo_hi = min(g.Wo - 1, floor_div(x0 + bw - 1 + R + g.pw, g.sw));
        }
        const int e_w = max(0, wo_hi - wo_lo + 1);
        const int e_cnt = e_w * max(0, ho_hi - ho_lo + 1);
        __syncthreads();
        // List the candidate pixels; four box reads per lane in flight.
        if (boxes_exact) {
            for (int e0 = warp * 128; e0 < e_cnt; e0 += nwarps * 128) {
                uint32_t box[4];
                int hos[4], wos[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + u * 32 + lane;
                    const int eh = e / e_w;
                    hos[u] = ho_lo + eh;
                    wos[u] = wo_lo + (e - eh * e_w);
                    box[u] = e < e_cnt ? boxes[pix0 + static_cast<long long>(hos[u]) * g.Wo + wos[u]] : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int bh0 = hos[u] * g.sh - g.ph, bw0 = wos[u] * g.sw - g.pw;
                    const int rmin = bh0 + static_cast<int8_t>(box[u] & 0xff);
                    const int rmax = bh0 + static_cast<int8_t>((box[u] >> 8) & 0xff);
                    const int cmin = bw0 + static_cast<int8_t>((box[u] >> 16) & 0xff);
                    const int cmax = bw0 + static_cast<int8_t>(box[u] >> 24);
                    const bool keep = e0 + u * 32 + lane < e_cnt && rmax >= y0 - 1 && rmin <= y0 + bh - 1 &&
                                      cmax >= x0 - 1 && cmin <= x0 + bw - 1;
                    const unsigned ball = __ballot_sync(0xffffffffu, keep);
                    int base = 0;
                    if (lane == 0 && ball) base = atomicAdd(&s_nlist, __popc(ball));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const int pos = base + __popc(ball & ((1u << lane) - 1));
                    if (keep && pos < kListCap)
                        s_list[pos] = (static_cast<uint32_t>(hos[u]) << 16) | static_cast<uint32_t>(wos[u]);
                }
            }
        }
        __syncthreads();
        const int nlist = s_nlist;
        sorted = boxes_exact && nlist <= kListCap && g.Ho <= 65535 && g.Wo <= 65535 && compact_ok &&
                 static_cast<long long>(g.Ho) * g.Wo * g.C < (1LL << 31);
        if (sorted) {
            // Each thread keeps one (group, point) -- its bin base and anchor
            // offset stay in registers -- and walks the listed pixels of its
            // slot, kScanBatch code reads in flight.  Pass 0 counts the samples
            // of each (group, cell); pass 1 places their records in bin order.
            const int spt = GK <= nthr ? nthr / GK : 1;
            const int tslot = GK <= nthr ? static_cast<int>(threadIdx.x) / GK : 0;
            const int gk_first = threadIdx.x - tslot * GK;
            const int Wo = g.Wo, sh = g.sh, sw = g.sw;
            for (int pass = 0; pass < 2; ++pass) {
                if (pass == 1) {
                    sorted = bins_exclusive_scan(cnt, cur, nbins, s_warp, &s_total) <= g.bcap;
                    if (!sorted) break;
                }
                for (int gk = gk_first; tslot < spt && gk < GK; gk += nthr) {
                    const int4 tb = s_tab[gk];
                    const long long ebase = pix0 * GK + gk;  // entry of listed pixel pix: ebase + pix * GK
                    const int sk = tb.w & 0xffff, sg = tb.w >> 16;
                    int ih, iw;
                    grid_cell_of(g, sk, ih, iw);
                    for (int e0 = tslot; e0 < nlist; e0 += kScanBatch * spt) {
                        // Cell of each sample: fp32 from its code; 16-bit dtypes
                        // re-form it from the offsets (the same fp32 fma).
                        uint32_t lv[kScanBatch];
                        int bin[kScanBatch];
                        Candidate c[kScanBatch];
#pragma unroll
                        for (int u = 0; u < kScanBatch; ++u) {
                            const int e = e0 + u * spt;
                            lv[u] = e < nlist ? s_list[e] : 0;
                            const int ho = static_cast<int>(lv[u] >> 16), wo = static_cast<int>(lv[u] & 0xffff);
                            const int pix = ho * Wo + wo;
                            c[u].any = false;
                            if (e < nlist) {
                                if constexpr (COMPACT) {
                                    c[u] = candidate(g, om + (pix0 + pix) * g.P + sg * 3 * g.K, sk, ho, wo, ih, iw);
                                } else {
                                    const uint32_t cd = ld_stream_u16(sa.code + ebase + static_cast<long long>(pix) * GK);
                                    c[u].any = cd != kCodeNone;
                                    c[u].h0 = ho * sh + tb.y + (y0 - 1) + static_cast<int8_t>(cd & 0xff);
                                    c[u].w0 = wo * sw + tb.z + (x0 - 1) + static_cast<int8_t>(cd >> 8);
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < kScanBatch; ++u) {
                            const int ch = c[u].h0 - (y0 - 1), cw = c[u].w0 - (x0 - 1);
                            const bool in = c[u].any && static_cast<unsigned>(ch) <= static_cast<unsigned>(bh) &&
                                            static_cast<unsigned>(cw) <= static_cast<unsigned>(bw);
                            bin[u] = in ? tb.x + ch * cells_w + cw : -1;
                        }
                        if (pass == 0) {
#pragma unroll
                            for (int u = 0; u < kScanBatch; ++u)
                                if (bin[u] >= 0) atomicAdd(&cnt[bin[u]], 1);
                            continue;
                        }
#pragma unroll
                        for (int u = 0; u < kScanBatch; ++u) {
                            if (bin[u] < 0) continue;
                            const int ho = static_cast<int>(lv[u] >> 16), wo = static_cast<int>(lv[u] & 0xffff);
                            const int pix = ho * Wo + wo;
                            const T* orow = om + (pix0 + pix) * g.P + sg * 3 * g.K;
                            const int slot = atomicAdd(&cur[bin[u]], 1);
                            if constexpr (COMPACT) {
                                uint32_t id;
                                if (!compact_source(ho, wo, ho_ref, wo_ref, id)) s_fail = 1;
                                const uint32_t mb =
                                    smax ? weight_q16(softmax_weight(to_f32(orow[2 * g.K + sk]), softmax_stats(orow + 2 * g.K, g.K)))
                                         : ld_stream_u16(orow + 2 * g.K + sk);
                                rec_c[slot] = make_uint2(id | (mb << 16), fix16(c[u].lh) | (fix16(c[u].lw) << 16));
                            } else {
                                const Candidate cc = candidate(g, orow, sk, ho, wo, ih, iw);
                                float mf = ld_stream_elem(orow + 2 * g.K + sk);
                                if (smax) mf = softmax_weight(mf, softmax_stats(orow + 2 * g.K, g.K));
                                const float b = mf * cc.lh;
                                rec_w[slot] = make_float4(__int_as_float(pix * g.C), mf - b, b, cc.lw);
                            }
                        }
                    }
                }
                __syncthreads();
            }
            if (sorted) sorted = s_fail == 0;
        }
    }

    if (sorted) {
        // Pull over strips.  A strip is LW lanes of a warp; lane cx owns cell
        // column cx of one (group, channel slice) and one segment of BS pixel
        // rows, and walks the segment's cell rows top to bottom.  Each sample
        // of its cell is read once and added, with its four bilinear weights,
        // to the partial sums of the cell's corners: left/right of the pixel
        // row above the cell (top) and of the row below it (bottom).  After a
        // cell row the pixel row above it is complete but for the left
        // corners of the next cell column, which the next lane holds: one
        // shuffle adds them and the lane writes its pixel.  Partial sums that
        // fall outside the segment are dropped (the neighbouring segment
        // forms them too).
        const int LW = g.LW;
        const int strips = 32 / LW;
        const int cx = lane & (LW - 1);
        const int gs_count = g.G * g.nslice;
        const int items = gs_count * g.nseg;
        for (int base = warp * strips; base < items; base += nwarps * strips) {
            const int item = base + lane / LW;
            const bool live = item < items;
            const int seg = item / gs_count;
            const int gsl = item - seg * gs_count;
            const int grp = gsl / g.nslice, sl = gsl - (gsl / g.nslice) * g.nslice;
            const int r0 = seg * g.BS;
            const int r1 = min(r0 + g.BS, bh);  // pixel rows [r0, r1) of the tile
            const int ch_off = grp * g.Cg + sl * (VEC * EPV);
            GySource<T> gs;
            gs.row = g.Wo * g.C;
            gs.col = g.C;
            gs.ref = gout + pix0 * g.C + ch_off;
            if constexpr (COMPACT) gs.ref += (static_cast<long long>(ho_ref - 64) * g.Wo + (wo_ref - 64)) * g.C;
            // Ping-pong partial sums: A and B alternate as the pixel row above
            // (top) and below (bottom) the current cell row.
            float2 a0[PAIRS], a1[PAIRS], b0[PAIRS], b1[PAIRS];
#pragma unroll
            for (int i = 0; i < PAIRS; ++i) a0[i] = a1[i] = b0[i] = b1[i] = make_float2(0.f, 0.f);
            const bool has_col = live && cx <= bw;
            T* dst_col = gvalue + ((static_cast<long long>(n) * g.H + y0) * g.W + x0 + cx) * g.C + ch_off;
            const long long row_stride = static_cast<long long>(g.W) * g.C;
            for (int t = 0; t <= g.BS; t += 2) {
                int cy = r0 + t;
                int end = 0, j = 0;
                if (has_col && cy <= r1) {
                    const int bin = grp * cells + cy * cells_w + cx;
                    end = cur[bin];
                    j = end - cnt[bin];
                }
                pull_cell<T, VEC, COMPACT>(rec_base, gs, smax, j, end, a0, a1, b0, b1);
                // pixel row cy - 1 (in A) is complete
                finish_row<T, VEC>(a0, a1, LW, live && t > 0 && cy - 1 < r1 && cx < bw, dst_col + (cy - 1) * row_stride);
                if (t + 1 > g.BS) break;
                ++cy;
                end = j = 0;
                if (has_col && cy <= r1) {
                    const int bin = grp * cells + cy * cells_w + cx;
                    end = cur[bin];
                    j = end - cnt[bin];
                }
                pull_cell<T, VEC, COMPACT>(rec_base, gs, smax, j, end, b0, b1, a0, a1);
                finish_row<T, VEC>(b0, b1, LW, live && cy - 1 < r1 && cx < bw, dst_col + (cy - 1) * row_stride);
            }
        }
        return;
    }

    // Direct path (records that do not fit, or a tile the sort cannot name):
    // thread -> (input pixel, group, slice) of the tile, scanning every
    // candidate sample of its group.
    if (threadIdx.x == 0) atomicAdd(sa.diag + kDiagDirect, 1);
    const int lanes_pp = g.G * g.nslice;
    const int uh_lo = max(0, ceil_div(y0 - R + g.ph - (g.kh - 1) * g.dh, g.sh));
    const int uh_hi = min(g.Ho - 1, floor_div(y0 + bh - 1 + R + g.ph, g.sh));
    const int uw_lo = max(0, ceil_div(x0 - R + g.pw - (g.kw - 1) * g.dw, g.sw));
    const int uw_hi = min(g.Wo - 1, floor_div(x0 + bw - 1 + R + g.pw, g.sw));
    const int u_w = max(0, uw_hi - uw_lo + 1);
    const int u_cnt = R >= 0 ? u_w * max(0, uh_hi - uh_lo + 1) : 0;
    for (int it = threadIdx.x; it < bh * bw * lanes_pp; it += nthr) {
        const int q = it / lanes_pp;
        const int rr = it - q * lanes_pp;
        const int grp = rr / g.nslice;
        const int sl = rr - grp * g.nslice;
        const int qy = q / bw, qx = q - (q / bw) * bw;
        const int ch_off = grp * g.Cg + sl * (VEC * EPV);
        const T* gy_img = gout + pix0 * g.C + ch_off;
        float2 acc[PAIRS];
#pragma unroll
        for (int i = 0; i < PAIRS; ++i) acc[i] = make_float2(0.f, 0.f);
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
                    float m = to_f32(orow[2 * g.K + k]);
                    if (smax) m = softmax_weight(m, softmax_stats(orow + 2 * g.K, g.K));
                    const float wt = m * (a ? c.lh : 1.f - c.lh) * (b ? c.lw : 1.f - c.lw);
                    accumulate<T, VEC>(acc, gy_img + static_cast<long long>(ho * g.Wo + wo) * g.C, wt);
                }
            }
        }
        T* dst = gvalue + ((static_cast<long long>(n) * g.H + gy_abs) * g.W + gx_abs) * g.C + ch_off;
        if constexpr (VEC == 2) {
            st_global32(dst, pack(acc, T()), pack(acc + EPV / 2, T()));
        } else {
            st_global(dst, pack(acc, T()));
        }
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

template <typename T, int VEC, int KH, int KW, bool RC, bool SM>
cudaError_t launch_samples_typed(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                                 int* reach, SampleArrays sa, uint32_t* boxes, cudaStream_t stream) {
    const size_t smem = backward_smem_bytes(g, sizeof(T));
    auto kern = samples_kernel<T, VEC, KH, KW, RC, SM>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const long long blocks = static_cast<long long>(g.N) * g.tiles_h * g.tiles_w;
    const int threads = samples_threads(g);
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(g, static_cast<const T*>(value),
                                                                   static_cast<const T*>(om), static_cast<const T*>(gout),
                                                                   static_cast<T*>(gom), reach, sa, boxes);
    return cudaGetLastError();
}

template <typename T, int VEC, bool SM>
cudaError_t launch_samples_grid(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                                int* reach, SampleArrays sa, uint32_t* boxes, cudaStream_t stream) {
    if (g.kh == 3 && g.kw == 3) {
        return g.remove_center
                   ? launch_samples_typed<T, VEC, 3, 3, true, SM>(g, value, om, gout, gom, reach, sa, boxes, stream)
                   : launch_samples_typed<T, VEC, 3, 3, false, SM>(g, value, om, gout, gom, reach, sa, boxes, stream);
    }
    return launch_samples_typed<T, VEC, 0, 0, false, SM>(g, value, om, gout, gom, reach, sa, boxes, stream);
}

template <typename T, int VEC>
cudaError_t launch_samples_softmax(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                                   int* reach, SampleArrays sa, uint32_t* boxes, cudaStream_t stream) {
    return g.softmax ? launch_samples_grid<T, VEC, true>(g, value, om, gout, gom, reach, sa, boxes, stream)
                     : launch_samples_grid<T, VEC, false>(g, value, om, gout, gom, reach, sa, boxes, stream);
}

template <typename T>
cudaError_t launch_samples_vec(const Geometry& g, const void* value, const void* om, const void* gout, void* gom,
                               int* reach, SampleArrays sa, uint32_t* boxes, cudaStream_t stream) {
    return g.vec == 2 ? launch_samples_softmax<T, 2>(g, value, om, gout, gom, reach, sa, boxes, stream)
                      : launch_samples_softmax<T, 1>(g, value, om, gout, gom, reach, sa, boxes, stream);
}

template <typename T, int VEC, bool SM>
cudaError_t launch_value_typed(const Geometry& g, const void* om, const void* gout, void* gvalue, const int* reach,
                               SampleArrays sa, const uint32_t* boxes, cudaStream_t stream) {
    const size_t smem = backward_value_smem_bytes(g);
    auto kern = value_kernel<T, VEC, sizeof(T) == 2, SM>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const long long blocks = static_cast<long long>(g.N) * g.btiles_h * g.btiles_w;
    kern<<<static_cast<unsigned>(blocks), g.bthreads, smem, stream>>>(
        g, static_cast<const T*>(om), static_cast<const T*>(gout), static_cast<T*>(gvalue), reach, sa, boxes);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_value_vec(const Geometry& g, const void* om, const void* gout, void* gvalue, const int* reach,
                             SampleArrays sa, const uint32_t* boxes, cudaStream_t stream) {
    if (g.softmax)
        return g.vec == 2 ? launch_value_typed<T, 2, true>(g, om, gout, gvalue, reach, sa, boxes, stream)
                          : launch_value_typed<T, 1, true>(g, om, gout, gvalue, reach, sa, boxes, stream);
    return g.vec == 2 ? launch_value_typed<T, 2, false>(g, om, gout, gvalue, reach, sa, boxes, stream)
                      : launch_value_typed<T, 1, false>(g, om, gout, gvalue, reach, sa, boxes, stream);
}

}  // namespace

size_t backward_smem_bytes(const Geometry& g, int elem_bytes) {
    size_t b = static_cast<size_t>(g.TH) * g.TW * g.P * elem_bytes * 2;
    if (elem_bytes == 2 && g.buckets) {  // staging: meta words only for the unrolled grids without softmax
        const size_t per = (g.kh == 3 && g.kw == 3 && !g.softmax && !g.remove_center) ? 8 : 16;
        b += static_cast<size_t>(filing_chunk(g)) * samples_threads(g) * per;
    }
    return b;
}

size_t backward_value_smem_bytes(const Geometry& g) {
    const size_t nbins = static_cast<size_t>(g.G) * (g.BH + 1) * (g.BW + 1);
    return ((2 * nbins + kListCap) * sizeof(int) + 15) / 16 * 16 + static_cast<size_t>(g.G) * g.K * sizeof(int4) +
           static_cast<size_t>(g.bcap) * g.brec;
}

cudaError_t launch_backward_samples(const Geometry& g, int dtype, const void* value, const void* om, const void* gout,
                                    void* gom, int* reach, SampleArrays sa, uint32_t* boxes, cudaStream_t stream) {
    switch (dtype) {
        case 0: return launch_samples_vec<float>(g, value, om, gout, gom, reach, sa, boxes, stream);
        case 1: return launch_samples_vec<__half>(g, value, om, gout, gom, reach, sa, boxes, stream);
        case 2: return launch_samples_vec<__nv_bfloat16>(g, value, om, gout, gom, reach, sa, boxes, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_backward_value(const Geometry& g, int dtype, const void* om, const void* gout, void* gvalue,
                                  const int* reach, SampleArrays sa, const uint32_t* boxes,
                                  cudaStream_t stream) {
    switch (dtype) {
        case 0: return launch_value_vec<float>(g, om, gout, gvalue, reach, sa, boxes, stream);
        case 1: return launch_value_vec<__half>(g, om, gout, gvalue, reach, sa, boxes, stream);
        case 2: return launch_value_vec<__nv_bfloat16>(g, om, gout, gvalue, reach, sa, boxes, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
