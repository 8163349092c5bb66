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
//
// Fused producer (LIN).  The DCNv4 module computes the offsets and dynamic
// weights with one merged linear layer (CSDN summary, section 2.2 "DCN模块的微设计"):
// offset_mask = x W^T + b.  With LIN the kernel stages the tile's rows of x
// instead (cp.async, double buffered), forms the tile's offset_mask rows on
// the tensor cores (mma.sync m16n8k16, fp32 accumulation, bias added, rounded
// once to the I/O dtype) into shared memory, optionally stores them, and
// samples them as above: the offset_mask never makes a round trip through HBM.
#include <algorithm>
#include <atomic>
#include <type_traits>

#include "dcn4_common.cuh"
#include "dcn4_tcgen05.cuh"

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
// offset_mask tiles in flight per CTA (plain and PROJ, g.fbufs): three when they still
// leave room for kFwdCtasPerSm CTAs an SM, else two.  With three, the buffer a tile is
// copied into was last read two tiles earlier, before a barrier every thread has since
// passed, so a tile needs one barrier, not two.
constexpr int kFwdMaxBufs = 3;

// Arguments of the fused producer: x [N, Ho, Wo, Cx], w [P, Cx] (nn.Linear
// layout), b [P] or null, om_out [N, Ho, Wo, P] or null; and of the fused
// output projection: pw [Cout, C], pb [Cout] or null, core_out [N, Ho, Wo, C]
// (the aggregation's own output) or null.
template <typename T>
struct LinearArgs {
    const T* x;
    const T* w;
    const T* b;
    T* om_out;
    int Cx;
    int w_smem;  // 1: W is staged in shared memory once per CTA (when it fits)
    int tc;      // 1: the offset_mask tile is formed on tcgen05 (see stage_x_swizzled)
    const T* pw;
    const T* pb;
    T* core_out;
    int Cout;
};

// tcgen05 form of the producer: D^T[p][pixel] = W x^T with M = 128 rows of W
// (P <= 128, the rest zero), N = the tile's 64 pixels, K = Cx in 64-wide slabs,
// the accumulator in tensor memory.  W and the x tiles sit in shared memory in
// the 128-byte swizzled K-major layout: row r of a slab at r*128 bytes, its
// 16-byte chunk c at ((c ^ (r % 8)) * 16), slabs of 64 columns one after the
// other.  The SMs' tensor cores form the tile while the warps only stage
// operands and read the result back into the tile's offset_mask rows.
constexpr int kTcRows = 128, kTcPix = 64;
__host__ __device__ inline int tc_x_bytes(int Cx) { return kTcPix * Cx * 2; }
__host__ __device__ inline int tc_w_bytes(int Cx) { return kTcRows * Cx * 2; }
__device__ unsigned g_fwd_linear_status;  // nonzero once a bounded wait of the tcgen05 producer gave up

// Output projection y = core W_out^T + b_out fused behind the sampler (PROJ): per
// tile D^T[o][pixel] = W_out core^T with M = 128 rows (Cout <= 128), N = the tile's
// pixels (16, 32 or 64), K = C in 64-wide slabs; the same swizzled K-major operand
// layout as the producer.  W_out keeps only its Cout rows per slab (slab stride
// Cout * 128 bytes): the MMA's rows past Cout read whatever follows (the next slab,
// the core tile), and those result rows are never read.  The core tile is written by
// the sampling threads themselves (their fp32 sums rounded to the I/O dtype, as the
// unfused pair stores them); once the MMAs have completed, the same memory takes
// the [pixels][Cout] result, which 16-byte writes store.  Every byte of shared
// memory kept small here is L1 left to the sampler's gathers.
__host__ __device__ inline int proj_slab_bytes(int Cout) { return Cout * 128; }
__host__ __device__ inline int proj_tile_bytes(const Geometry& g, int Cout) {
    return g.pix_per_cta * (g.C > Cout ? g.C : Cout) * 2;  // the core tile, then the result tile
}
__host__ __device__ inline int proj_tmem_cols(const Geometry& g) { return g.pix_per_cta < 32 ? 32 : g.pix_per_cta; }
// W_out's slabs, the shared tile and the bias, and at least as far as the last slab's
// 128-row operand reads.
__host__ __device__ inline int proj_area_bytes(const Geometry& g, int Cout) {
    const int nslab = g.C / 64, slab = proj_slab_bytes(Cout);
    const int body = nslab * slab + proj_tile_bytes(g, Cout) + Cout * static_cast<int>(sizeof(float));
    const int reach = (nslab - 1) * slab + kTcRows * 128;
    return body > reach ? body : reach;
}
// Shared memory of the projection beyond the offset_mask tiles and exponentials
// (with the 1024-byte alignment slack of the swizzled operands).
inline size_t proj_extra_bytes(const Geometry& g, int Cout) { return 1024 + static_cast<size_t>(proj_area_bytes(g, Cout)); }
// The softmax exponentials [K][threads] (fp32), when the masks are logits.
inline size_t forward_exps_bytes(const Geometry& g) {
    return g.softmax ? static_cast<size_t>(g.K) * samples_threads(g) * sizeof(float) : 0;
}
// offset_mask tiles per CTA for a CTA that also holds `extra` bytes (see kFwdMaxBufs).
inline int forward_bufs(const Geometry& g, int elem_bytes, size_t extra) {
    const size_t tile = static_cast<size_t>(g.pix_per_cta) * g.P * elem_bytes;
    return kFwdMaxBufs * tile + forward_exps_bytes(g) + extra + 1024 <= 227 * 1024 / kFwdCtasPerSm ? kFwdMaxBufs : 2;
}

// Rows of a staged x tile: the tile's pixels rounded up to whole 16-row MMA tiles.
__host__ __device__ inline int linear_rows(const Geometry& g) { return (g.TH * g.TW + 15) / 16 * 16; }
// Elements per staged x (and W) row: 8 of padding keep ldmatrix's eight row reads on distinct banks.
__host__ __device__ inline int linear_ld(int Cx) { return Cx + 8; }
// Column tiles (of 8 outputs) one GEMM item covers.
constexpr int kLinNB = 4;
// Rows of a staged W: whole items of kLinNB column tiles.
__host__ __device__ inline int linear_w_rows(const Geometry& g) { return (g.P / 8 + kLinNB - 1) / kLinNB * kLinNB * 8; }

__device__ __forceinline__ void ldmatrix_x4(uint32_t* r, unsigned addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += a (16x16, row-major fragment) * b (16x8, column fragment), fp32 accumulation.
template <typename T>
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, const uint32_t* b) {
    if constexpr (std::is_same<T, __half>::value) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                     "{%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    } else {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                     "{%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    }
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    uint32_t u;
    if constexpr (std::is_same<T, __half>::value) {
        const __half2 h = __floats2half2_rn(lo, hi);
        memcpy(&u, &h, 4);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        memcpy(&u, &h, 4);
    }
    return u;
}

// The tile's rows of x, swizzled for tcgen05 (see kTcRows), with cp.async.
template <typename T>
__device__ __forceinline__ void stage_x_swizzled(uint32_t dst, const LinearArgs<T>& lin, const Geometry& g,
                                                 const Tile& t) {
    const int cpp = lin.Cx / 8;  // 16-byte chunks per pixel
    const int total = t.th * t.tw * cpp;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int q = i / cpp, c = i - q * cpp;
        const int py = q / t.tw, px = q - py * t.tw;
        const int row = py * g.TW + px;
        const long long pix = (static_cast<long long>(t.n) * g.Ho + t.ho0 + py) * g.Wo + t.wo0 + px;
        const T* sp = lin.x + pix * lin.Cx + c * 8;
        const uint32_t d = dst + (c >> 3) * (kTcPix * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(sp));
    }
    asm volatile("cp.async.commit_group;");
}

// The tile's rows of x into shared memory [rows][Cx + 8] with cp.async.
template <typename T>
__device__ __forceinline__ void stage_x_async(T* dst, const LinearArgs<T>& lin, const Geometry& g, const Tile& t) {
    constexpr int EPV = Elem<T>::per16;
    const int cpp = lin.Cx / EPV;  // 16-byte chunks per pixel
    const int total = t.th * t.tw * cpp;
    const int ld = linear_ld(lin.Cx);
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int q = i / cpp, c = i - q * cpp;
        const int py = q / t.tw, px = q - py * t.tw;
        const long long pix = (static_cast<long long>(t.n) * g.Ho + t.ho0 + py) * g.Wo + t.wo0 + px;
        const T* sp = lin.x + pix * lin.Cx + c * EPV;
        T* d = dst + (py * g.TW + px) * ld + c * EPV;
        const unsigned da = static_cast<unsigned>(__cvta_generic_to_shared(d));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(da), "l"(sp));
    }
    asm volatile("cp.async.commit_group;");
}

template <typename T>
__device__ __forceinline__ void store_pair_rows(T* om_s, const Geometry& g, int rows, int mt, int col, const float* acc,
                                                const float* b_s) {
    const int lane = threadIdx.x & 31;
    const float2 bb = *reinterpret_cast<const float2*>(b_s + col);
    const int r0 = mt * 16 + (lane >> 2), r1 = r0 + 8;
    if (r0 < rows) *reinterpret_cast<uint32_t*>(om_s + r0 * g.P + col) = pack2<T>(acc[0] + bb.x, acc[1] + bb.y);
    if (r1 < rows) *reinterpret_cast<uint32_t*>(om_s + r1 * g.P + col) = pack2<T>(acc[2] + bb.x, acc[3] + bb.y);
}

// om_s = round(x_s W^T + b) with W staged and KS = Cx / 16 k-steps known at
// compile time: a warp keeps one 16-row tile's A fragments for all k-steps in
// registers and walks its share of the 8-column tiles, loading each tile's B
// fragments two k-steps per ldmatrix.
template <typename T, int KS>
__device__ __forceinline__ void linear_tile_staged(const Geometry& g, const LinearArgs<T>& lin, const T* x_s,
                                                   const T* w_s, T* om_s, const float* b_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int rows = g.TH * g.TW;
    const int MT = linear_rows(g) / 16, NT = g.P / 8;
    const int ld = linear_ld(lin.Cx);
    const int wpm = max(1, nw / MT);  // warps per 16-row tile
    const int sub = warp % wpm;
    for (int mt = warp / wpm; mt < MT; mt += nw / wpm) {
        uint32_t a[KS][4];
        const unsigned a_addr =
            static_cast<unsigned>(__cvta_generic_to_shared(x_s + (mt * 16 + (lane & 15)) * ld + (lane >> 4) * 8));
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) ldmatrix_x4(a[ks], a_addr + ks * 32);
        // lane l: row l % 8 of the column tile, k offset 8 * (l / 8) within two k-steps
        const unsigned b_base =
            static_cast<unsigned>(__cvta_generic_to_shared(w_s + (lane & 7) * ld + (lane >> 3) * 8));
        for (int nt = sub; nt < NT; nt += wpm) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const unsigned b_addr = b_base + nt * 8 * ld * 2;
#pragma unroll
            for (int ks = 0; ks < KS; ks += 2) {
                uint32_t b[4];
                if constexpr (KS == 1) {
                    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                                 : "=r"(b[0]), "=r"(b[1])
                                 : "r"(b_addr));
                } else {
                    ldmatrix_x4(b, b_addr + ks * 32);
                }
                mma_16816<T>(acc, a[ks], b);
                if constexpr (KS > 1) mma_16816<T>(acc, a[ks + 1], b + 2);
            }
            store_pair_rows<T>(om_s, g, rows, mt, nt * 8 + (lane & 3) * 2, acc, b_s);
        }
    }
}

// om_s [TH*TW][P] = round(x_s W^T + b) for the tile: warps take (16-row tile,
// 4 column tiles of 8) items; A fragments come from shared memory (ldmatrix),
// B fragments from the staged W (ldmatrix, two column tiles per instruction)
// or, when W does not fit shared memory, straight from global memory.
template <typename T>
__device__ __forceinline__ void linear_tile(const Geometry& g, const LinearArgs<T>& lin, const T* x_s, const T* w_s,
                                            T* om_s, const float* b_s) {
    constexpr int NB = kLinNB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int rows = g.TH * g.TW;
    const int MT = linear_rows(g) / 16, NT = g.P / 8, KS = lin.Cx / 16;
    const int NCH = (NT + NB - 1) / NB;
    const int ld = linear_ld(lin.Cx);
    const int gq = lane >> 2, tq = lane & 3;
    for (int item = warp; item < MT * NCH; item += nw) {
        const int mt = item / NCH, nt0 = (item - mt * NCH) * NB;
        float acc[NB][4];
#pragma unroll
        for (int j = 0; j < NB; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        // lane l reads row l % 16 of the 16-row tile, column half l / 16
        const unsigned a_addr =
            static_cast<unsigned>(__cvta_generic_to_shared(x_s + (mt * 16 + (lane & 15)) * ld + (lane >> 4) * 8));
        if (lin.w_smem) {
            // lanes 0-7 / 8-15: rows of column tile nt, k halves 0 / 1; lanes 16-31: column tile nt + 1
            const int brow = (lane & 7) + ((lane >> 4) << 3), bcol = ((lane >> 3) & 1) * 8;
            const unsigned b_addr = static_cast<unsigned>(__cvta_generic_to_shared(w_s + (nt0 * 8 + brow) * ld + bcol));
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a[4], b[NB / 2][4];
                ldmatrix_x4(a, a_addr + ks * 32);
#pragma unroll
                for (int jj = 0; jj < NB / 2; ++jj) ldmatrix_x4(b[jj], b_addr + (jj * 16 * ld + ks * 16) * 2);
#pragma unroll
                for (int j = 0; j < NB; ++j)
                    if (nt0 + j < NT) mma_16816<T>(acc[j], a, &b[j >> 1][(j & 1) * 2]);  // uniform over the warp
            }
        } else {
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a[4];
                ldmatrix_x4(a, a_addr + ks * 32);
#pragma unroll
                for (int j = 0; j < NB; ++j) {
                    if (nt0 + j >= NT) break;  // uniform over the warp
                    const T* wr = lin.w + static_cast<long long>((nt0 + j) * 8 + gq) * lin.Cx + ks * 16 + tq * 2;
                    const uint32_t b[2] = {__ldg(reinterpret_cast<const unsigned*>(wr)),
                                           __ldg(reinterpret_cast<const unsigned*>(wr + 8))};
                    mma_16816<T>(acc[j], a, b);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            if (nt0 + j >= NT) break;
            const int col = (nt0 + j) * 8 + tq * 2;
            const float b0 = b_s[col], b1 = b_s[col + 1];
            const int r0 = mt * 16 + gq, r1 = r0 + 8;
            if (r0 < rows) *reinterpret_cast<uint32_t*>(om_s + r0 * g.P + col) = pack2<T>(acc[j][0] + b0, acc[j][1] + b1);
            if (r1 < rows) *reinterpret_cast<uint32_t*>(om_s + r1 * g.P + col) = pack2<T>(acc[j][2] + b0, acc[j][3] + b1);
        }
    }
}

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
// tile + gridDim.x, ...), copying the next tile's offset_mask rows (LIN: x
// rows) into the other half of a double buffer (cp.async) while it computes
// the current one.  KH, KW > 0: compile-time grid size (fully unrolled) and
// RC = remove_center; KH = KW = 0: sizes and remove_center from g.  SM:
// softmax over the K masks.  LIN: offset_mask rows from the linear producer.
// PROJ: the output projection behind the sampler (see proj_slab_bytes).
template <typename T, int VEC, int KH, int KW, bool RC, bool SM, bool LIN, bool PROJ>
__global__ void __launch_bounds__(256, kFwdCtasPerSm) forward_kernel(const Geometry g, const T* __restrict__ value,
                                                      const T* __restrict__ om, T* __restrict__ out,
                                                      const LinearArgs<T> lin) {
    static_assert(!(LIN && PROJ), "the producer and the projection are separate instantiations");
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int EPV = Elem<T>::per16;
    constexpr int PAIRS = VEC * EPV / 2;
    const int tile_elems = g.TH * g.TW * g.P;
    // plain: g.fbufs offset_mask tiles, the exponentials; LIN: one offset_mask tile, two x
    // tiles, W (when staged), the bias (fp32); PROJ: as plain, then the projection's tiles
    T* om_buf;  // the first offset_mask tile (plain and PROJ: g.fbufs of them follow one another)
    T* xbuf[2] = {nullptr, nullptr};
    T* w_s = nullptr;
    float* b_s = nullptr;
    float* e_s;  // softmax exponentials [K][threads]
    // tcgen05 producer: shared addresses of the two swizzled x tiles and of W (1024-byte aligned)
    const uint32_t sbase = tc::smem_u32(smem);
    uint32_t tc_x[2] = {0u, 0u}, tc_w = 0u;
    __shared__ __align__(8) uint64_t tc_mbar;
    __shared__ uint32_t tc_taddr;
    __shared__ int tc_abort;
    if constexpr (LIN) {
        om_buf = reinterpret_cast<T*>(smem);
        if (lin.tc) {
            tc_x[0] = (sbase + static_cast<uint32_t>(tile_elems) * 2u + 1023u) & ~1023u;
            tc_x[1] = tc_x[0] + tc_x_bytes(lin.Cx);
            tc_w = tc_x[1] + tc_x_bytes(lin.Cx);
            b_s = reinterpret_cast<float*>(smem + (tc_w - sbase) + tc_w_bytes(lin.Cx));
        } else {
            const int xs = linear_rows(g) * linear_ld(lin.Cx);
            xbuf[0] = om_buf + tile_elems;
            xbuf[1] = xbuf[0] + xs;
            w_s = xbuf[1] + xs;
            b_s = reinterpret_cast<float*>(w_s + (lin.w_smem ? linear_w_rows(g) * linear_ld(lin.Cx) : 0));
        }
        e_s = b_s + g.P;
    } else {
        om_buf = reinterpret_cast<T*>(smem);
        e_s = reinterpret_cast<float*>(om_buf + g.fbufs * tile_elems);
    }
    // PROJ: W_out's swizzled slabs (1024-byte aligned), the swizzled core tile (later the
    // [pixels][Cout] result tile) and the bias (fp32), after the exponentials
    uint32_t pj_a = 0u, pj_w = 0u;
    T* pj_o = nullptr;
    float* pj_b = nullptr;
    if constexpr (PROJ) {
        const uint32_t end = sbase + static_cast<uint32_t>(g.fbufs * tile_elems * sizeof(T)) +
                             (SM ? static_cast<uint32_t>(g.K * blockDim.x * sizeof(float)) : 0u);
        pj_w = (end + 1023u) & ~1023u;
        pj_a = pj_w + (g.C / 64) * proj_slab_bytes(lin.Cout);  // Cout * 128 is a multiple of 2048
        pj_o = reinterpret_cast<T*>(smem + (pj_a - sbase));
        pj_b = reinterpret_cast<float*>(smem + (pj_a - sbase) + proj_tile_bytes(g, lin.Cout));
    }
    const int ntiles = g.N * g.tiles_h * g.tiles_w;
    int tile = blockIdx.x;
    if (tile >= ntiles) return;
    if constexpr (PROJ) {
        for (int j = threadIdx.x; j < lin.Cout; j += blockDim.x) pj_b[j] = lin.pb ? to_f32(lin.pb[j]) : 0.f;
        // W_out rows [Cout][C] into 64-wide swizzled slabs of Cout rows
        const int cpr = g.C / 8;
        for (int i = threadIdx.x; i < lin.Cout * cpr; i += blockDim.x) {
            const int r = i / cpr, c = i - r * cpr;
            *reinterpret_cast<uint4*>(smem + (pj_w - sbase) + (c >> 3) * proj_slab_bytes(lin.Cout) + r * 128 +
                                      (((c & 7) ^ (r & 7)) << 4)) =
                ld_gather(lin.pw + static_cast<long long>(r) * g.C + c * 8);
        }
        if (threadIdx.x == 0) {
            tc::mbar_init(tc::smem_u32(&tc_mbar), 1);
            tc_abort = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (threadIdx.x < 32) {  // proj_tmem_cols fp32 columns x 128 lanes: the accumulator
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             tc::smem_u32(&tc_taddr)),
                         "r"(proj_tmem_cols(g)));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        tc::tc_fence_before();
    }
    if constexpr (LIN) {
        for (int j = threadIdx.x; j < g.P; j += blockDim.x) b_s[j] = lin.b ? to_f32(lin.b[j]) : 0.f;
        if (lin.tc) {
            // W rows [P][Cx] into 64-wide swizzled slabs; rows P..127 zero (their results are never stored)
            const int cpr = lin.Cx / 8;
            for (int i = threadIdx.x; i < kTcRows * cpr; i += blockDim.x) {
                const int r = i / cpr, c = i - r * cpr;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < g.P) v = ld_gather(lin.w + static_cast<long long>(r) * lin.Cx + c * 8);
                *reinterpret_cast<uint4*>(smem + (tc_w - sbase) + (c >> 3) * (kTcRows * 128) + r * 128 +
                                          (((c & 7) ^ (r & 7)) << 4)) = v;
            }
            if (threadIdx.x == 0) {
                tc::mbar_init(tc::smem_u32(&tc_mbar), 1);
                tc_abort = 0;
                asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            }
            if (threadIdx.x < 32) {  // kTcPix fp32 columns x 128 lanes: the accumulator
                asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                                 tc::smem_u32(&tc_taddr)),
                             "r"(kTcPix));
                asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
            }
            tc::tc_fence_before();
            stage_x_swizzled(tc_x[0], lin, g, tile_at(g, tile));
        } else if (lin.w_smem) {  // W rows [P][Cx] -> [rows][Cx + 8]; rows past P stay unset (their columns are dropped)
            const int cpr = lin.Cx / EPV;
            for (int i = threadIdx.x; i < g.P * cpr; i += blockDim.x) {
                const int r = i / cpr, c = i - r * cpr;
                *reinterpret_cast<uint4*>(w_s + r * linear_ld(lin.Cx) + c * EPV) =
                    ld_gather(lin.w + static_cast<long long>(r) * lin.Cx + c * EPV);
            }
        }
        if (!lin.tc) stage_x_async(xbuf[0], lin, g, tile_at(g, tile));
    } else {
        stage_tile_async(om_buf, om, g, tile_at(g, tile));
    }

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

    int cur = 0;  // the buffer of this tile's offset_mask rows (plain and PROJ)
    for (int it = 0; tile < ntiles; ++it, tile += gridDim.x) {
        const int next = tile + gridDim.x;
        const int nxt = cur + 1 == g.fbufs ? 0 : cur + 1;
        if (next < ntiles) {
            if constexpr (LIN) {
                if (lin.tc) {
                    stage_x_swizzled(tc_x[(it + 1) & 1], lin, g, tile_at(g, next));
                } else {
                    stage_x_async(xbuf[(it + 1) & 1], lin, g, tile_at(g, next));
                }
            } else {
                stage_tile_async(reinterpret_cast<T*>(smem) + nxt * tile_elems, om, g, tile_at(g, next));
            }
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        // the tensor cores read the x tile through the async proxy
        if constexpr (LIN) {
            if (lin.tc) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncthreads();
        const Tile t = tile_at(g, tile);
        // the tile's rows, addressed from smem directly so the reads stay shared-space loads
        const T* om_s = reinterpret_cast<const T*>(smem) + (LIN ? 0 : cur * tile_elems);
        if constexpr (LIN) {
            if (lin.tc) {
                // one thread issues the tile's MMAs; all wait for them, then read the accumulator back:
                // warp w reads TMEM lanes (rows p) 32 (w % 4) .. + 31, pixel columns 32 (w / 4) .. + 31
                tc::tc_fence_after();
                const uint32_t tmem = tc_taddr;
                if (threadIdx.x == 0) {
                    constexpr uint32_t idesc = tc::umma_idesc<T>(kTcRows, kTcPix, 0, 0);
                    const uint32_t xb = tc_x[it & 1];
                    for (int sb = 0; sb < lin.Cx / 64; ++sb)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            tc::umma_f16(tmem, tc::umma_desc_sw128(tc_w + sb * (kTcRows * 128) + q * 32, 16, 1024),
                                         tc::umma_desc_sw128(xb + sb * (kTcPix * 128) + q * 32, 16, 1024), idesc,
                                         sb > 0 || q > 0);
                    tc::umma_commit(tc::smem_u32(&tc_mbar));
                }
                tc::mbar_wait_or(tc::smem_u32(&tc_mbar), static_cast<uint32_t>(it) & 1u, &tc_abort);
                tc::tc_fence_after();
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
                const int sub = warp & 3, half = warp >> 2;
                uint32_t acc32[32];
                tc::tmem_ld32(tmem + (static_cast<uint32_t>(32 * sub) << 16) + half * 32, acc32);
                const int pr = 32 * sub + lane;
                if (pr < g.P && !tc_abort) {
                    const float bp = b_s[pr];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        om_buf[(half * 32 + j) * g.P + pr] = from_f32<T>(__uint_as_float(acc32[j]) + bp);
                }
                tc::tc_fence_before();  // the next tile's MMAs overwrite the accumulator after the next barrier
            } else {
                switch (lin.w_smem ? lin.Cx / 16 : 0) {
                    case 1: linear_tile_staged<T, 1>(g, lin, xbuf[it & 1], w_s, om_buf, b_s); break;
                    case 2: linear_tile_staged<T, 2>(g, lin, xbuf[it & 1], w_s, om_buf, b_s); break;
                    case 4: linear_tile_staged<T, 4>(g, lin, xbuf[it & 1], w_s, om_buf, b_s); break;
                    case 8: linear_tile_staged<T, 8>(g, lin, xbuf[it & 1], w_s, om_buf, b_s); break;
                    default: linear_tile(g, lin, xbuf[it & 1], w_s, om_buf, b_s);
                }
            }
            __syncthreads();
            if (lin.tc && tc_abort) {  // a wait gave up: no further tile is formed
                if (threadIdx.x == 0) atomicOr(&g_fwd_linear_status, 1u);
                break;
            }
            if (lin.om_out) {  // the rows the samples use, 16-byte stores
                const int cpp = g.P / EPV;
                for (int i = threadIdx.x; i < t.th * t.tw * cpp; i += blockDim.x) {
                    const int q = i / cpp, c = i - q * cpp;
                    const int qy = q / t.tw, qx = q - qy * t.tw;
                    const long long pix = (static_cast<long long>(t.n) * g.Ho + t.ho0 + qy) * g.Wo + t.wo0 + qx;
                    st_global(lin.om_out + pix * g.P + c * EPV,
                              *reinterpret_cast<const uint4*>(om_buf + (qy * g.TW + qx) * g.P + c * EPV));
                }
            }
        }
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
            if constexpr (KH > 0) {
                // Compile-time grid: two-stage pipeline.  The four corner slices of
                // sample k + 1 are requested before the FMAs of sample k, so each
                // thread keeps eight 32-byte loads in flight instead of four.
                constexpr int KK = KH * KW - (RC ? 1 : 0);
                uint4 raw[2][4][VEC];
                float wts[2][4];
                auto issue = [&](int kk, int ih, int iw, uint4 (&r)[4][VEC], float (&wt)[4]) {
                    const float dx = to_f32(row[2 * kk]);
                    const float dy = to_f32(row[2 * kk + 1]);
                    float m = to_f32(row[2 * K + kk]);
                    if constexpr (SM) m = e_s[kk * blockDim.x + threadIdx.x] * inv;
                    const float h = __fmaf_rn(g.s, dy, static_cast<float>(hb + ih * g.dh));
                    const float w = __fmaf_rn(g.s, dx, static_cast<float>(wb + iw * g.dw));
                    const Cell<T> cell = bilinear_cell(g, img, h, w);
                    const float b = m * cell.lh, a = m - b;
                    const float wl = 1.f - cell.lw;
                    wt[0] = a * wl;
                    wt[1] = a * cell.lw;
                    wt[2] = b * wl;
                    wt[3] = b * cell.lw;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if constexpr (VEC == 2) {
                            ld_gather32(cell.c[c], r[c][0], r[c][1]);
                        } else {
                            r[c][0] = ld_gather(cell.c[c]);
                        }
                    }
                };
                auto consume = [&](const uint4 (&r)[4][VEC], const float (&wt)[4]) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 w2 = make_float2(wt[c], wt[c]);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            float2 f[EPV / 2];
                            unpack(r[c][v], f, T());
#pragma unroll
                            for (int i = 0; i < EPV / 2; ++i)
                                acc[v * (EPV / 2) + i] = __ffma2_rn(w2, f[i], acc[v * (EPV / 2) + i]);
                        }
                    }
                };
                // point kk -> grid cell (ih, iw): columns outer, rows inner, centre skipped
                auto cell_of = [](int kk, int& ih, int& iw) {
                    int idx = kk;
                    if (RC && idx >= (KW / 2) * KH + KH / 2) ++idx;
                    iw = idx / KH;
                    ih = idx - iw * KH;
                };
                {
                    int ih, iw;
                    cell_of(0, ih, iw);
                    issue(0, ih, iw, raw[0], wts[0]);
                }
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    if (kk + 1 < KK) {
                        int ih, iw;
                        cell_of(kk + 1, ih, iw);
                        issue(kk + 1, ih, iw, raw[(kk + 1) & 1], wts[(kk + 1) & 1]);
                    }
                    consume(raw[kk & 1], wts[kk & 1]);
                }
            } else {
                int k = 0;
                for (int iw = 0; iw < kw; ++iw) {
                    const float wbase = static_cast<float>(wb + iw * g.dw);
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
            }
            const long long o_off = ((static_cast<long long>(t.n) * g.Ho + ho) * g.Wo + wo) * g.C + ch_off;
            if constexpr (PROJ) {
                // the rounded sums into row lp of the swizzled core tile, 8 channels a chunk
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const uint4 q = pack(acc + v * (EPV / 2), T());
                    const int c = ch_off / 8 + v;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     pj_a + (c >> 3) * (g.pix_per_cta * 128) + lp * 128 + (((c & 7) ^ (lp & 7)) << 4)),
                                 "r"(q.x), "r"(q.y), "r"(q.z), "r"(q.w)
                                 : "memory");
                    if (lin.core_out) st_global(lin.core_out + o_off + v * EPV, q);
                }
            } else if constexpr (VEC == 2) {
                st_global32(out + o_off, pack(acc, T()), pack(acc + EPV / 2, T()));
            } else {
                st_global(out + o_off, pack(acc, T()));
            }
        } else if (PROJ && lp < g.pix_per_cta) {
            // a pixel past the image edge: its row is zero (its column of the result is not stored)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                const int c = ch_off / 8 + v;
                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(
                                 pj_a + (c >> 3) * (g.pix_per_cta * 128) + lp * 128 + (((c & 7) ^ (lp & 7)) << 4)),
                             "r"(0u)
                             : "memory");
            }
        }
        if constexpr (PROJ) {
            // the core tile is complete: one thread issues the MMAs, all wait, then the warps read the
            // accumulator back (warp w: TMEM lanes = rows o 32 (w % 4) .. + 31, pixel columns 32 (w / 4) ..)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            const uint32_t tmem = tc_taddr;
            const int npix = g.pix_per_cta;
            if (threadIdx.x == 0) {
                tc::tc_fence_after();
                const uint32_t idesc = tc::umma_idesc<T>(kTcRows, npix, 0, 0);
                for (int sb = 0; sb < g.C / 64; ++sb)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        tc::umma_f16(tmem, tc::umma_desc_sw128(pj_w + sb * proj_slab_bytes(lin.Cout) + q * 32, 16, 1024),
                                     tc::umma_desc_sw128(pj_a + sb * (npix * 128) + q * 32, 16, 1024), idesc,
                                     sb > 0 || q > 0);
                tc::umma_commit(tc::smem_u32(&tc_mbar));
            }
            tc::mbar_wait_or(tc::smem_u32(&tc_mbar), static_cast<uint32_t>(it) & 1u, &tc_abort);
            tc::tc_fence_after();
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            const int sub = warp & 3, half = warp >> 2;
            const int o = 32 * sub + lane;
            for (int j0 = half * 32; j0 < half * 32 + 32 && j0 < npix; j0 += 16) {  // whole warps
                uint32_t acc16[16];
                tc::tmem_ld16(tmem + (static_cast<uint32_t>(32 * sub) << 16) + j0, acc16);
                if (o < lin.Cout && !tc_abort) {
                    const float bo = pj_b[o];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pj_o[(j0 + j) * lin.Cout + o] = from_f32<T>(__uint_as_float(acc16[j]) + bo);
                }
            }
            tc::tc_fence_before();  // the next tile's MMAs overwrite the accumulator after the next barrier
            __syncthreads();
            if (tc_abort) {  // a wait gave up: no further tile is formed
                if (threadIdx.x == 0) atomicOr(&g_fwd_linear_status, 1u);
                break;
            }
            const int cpp = lin.Cout / EPV;  // the tile's y rows, 16-byte stores
            for (int i = threadIdx.x; i < t.th * t.tw * cpp; i += blockDim.x) {
                const int q = i / cpp, c = i - q * cpp;
                const int qy = q / t.tw, qx = q - qy * t.tw;
                const long long pix = (static_cast<long long>(t.n) * g.Ho + t.ho0 + qy) * g.Wo + t.wo0 + qx;
                st_global(out + pix * lin.Cout + c * EPV,
                          *reinterpret_cast<const uint4*>(pj_o + (qy * g.TW + qx) * lin.Cout + c * EPV));
            }
        }
        // Plain with two buffers: the next tile's copy (issued before the next top barrier) goes
        // to the buffer read two tiles ago only with three, so with two a barrier must come first.
        // LIN and PROJ need none here: LIN's next copies go to x buffers whose last reads precede
        // the post-GEMM barrier, and its om_s is rewritten only after the next top barrier; PROJ
        // reads om_s only before its first barrier, which precedes its second.
        if (!LIN && !PROJ && g.fbufs < 3) __syncthreads();
        cur = nxt;
    }
    if constexpr (PROJ) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        tc::tc_fence_before();
        __syncthreads();
        if (threadIdx.x < 32)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tc_taddr),
                         "r"(proj_tmem_cols(g)));
    }
    if constexpr (LIN) {
        if (lin.tc) {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            tc::tc_fence_before();
            __syncthreads();
            if (threadIdx.x < 32)
                asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tc_taddr), "r"(kTcPix));
        }
    }
}

template <typename T, int VEC, int KH, int KW, bool RC, bool SM, bool LIN, bool PROJ>
cudaError_t launch_typed(const Geometry& g, const void* value, const void* om, void* out, const LinearArgs<T>& lin,
                         cudaStream_t stream) {
    const size_t smem = LIN    ? forward_linear_smem_bytes(g, lin.Cx, lin.tc ? 2 : lin.w_smem ? 1 : 0)
                        : PROJ ? forward_proj_smem_bytes(g, lin.Cout)
                               : forward_smem_bytes(g, sizeof(T));
    Geometry gk = g;
    // PROJ keeps two offset_mask tiles: its own tiles already take shared memory, and what is
    // left is L1 for the gathers (a third tile was measured slower on every workload)
    gk.fbufs = LIN ? 1 : PROJ ? 2 : forward_bufs(g, sizeof(T), 0);
    auto kern = forward_kernel<T, VEC, KH, KW, RC, SM, LIN, PROJ>;
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
    kern<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        gk, static_cast<const T*>(value), static_cast<const T*>(om), static_cast<T*>(out), lin);
    return cudaGetLastError();
}

template <typename T, int VEC, bool SM, bool LIN, bool PROJ>
cudaError_t launch_grid(const Geometry& g, const void* value, const void* om, void* out, const LinearArgs<T>& lin,
                        cudaStream_t stream) {
    if (g.kh == 3 && g.kw == 3) {
        return g.remove_center ? launch_typed<T, VEC, 3, 3, true, SM, LIN, PROJ>(g, value, om, out, lin, stream)
                               : launch_typed<T, VEC, 3, 3, false, SM, LIN, PROJ>(g, value, om, out, lin, stream);
    }
    return launch_typed<T, VEC, 0, 0, false, SM, LIN, PROJ>(g, value, om, out, lin, stream);
}

template <typename T, int VEC, bool LIN, bool PROJ>
cudaError_t launch_softmax(const Geometry& g, const void* value, const void* om, void* out, const LinearArgs<T>& lin,
                           cudaStream_t stream) {
    return g.softmax ? launch_grid<T, VEC, true, LIN, PROJ>(g, value, om, out, lin, stream)
                     : launch_grid<T, VEC, false, LIN, PROJ>(g, value, om, out, lin, stream);
}

template <typename T, bool LIN = false, bool PROJ = false>
cudaError_t launch_vec(const Geometry& g, int vec, const void* value, const void* om, void* out,
                       const LinearArgs<T>& lin, cudaStream_t stream) {
    return vec == 2 ? launch_softmax<T, 2, LIN, PROJ>(g, value, om, out, lin, stream)
                    : launch_softmax<T, 1, LIN, PROJ>(g, value, om, out, lin, stream);
}

}  // namespace

size_t forward_linear_smem_bytes(const Geometry& g, int Cx, int mode) {
    const size_t om = static_cast<size_t>(g.pix_per_cta) * g.P * 2;  // 16-bit dtypes only
    const size_t tail = static_cast<size_t>(g.P) * sizeof(float) +
                        (g.softmax ? static_cast<size_t>(g.K) * samples_threads(g) * sizeof(float) : 0);
    if (mode == 2) return om + 1024 + 2 * static_cast<size_t>(tc_x_bytes(Cx)) + tc_w_bytes(Cx) + tail;
    const size_t xs = static_cast<size_t>(linear_rows(g)) * linear_ld(Cx) * 2;
    const size_t ws = mode == 1 ? static_cast<size_t>(linear_w_rows(g)) * linear_ld(Cx) * 2 : 0;
    return om + 2 * xs + ws + tail;
}

int forward_linear_mode(const Geometry& g, int Cx) {
    // Both need the CTA to still fit three to an SM (the sampler's occupancy).
    const size_t budget = 227 * 1024 / kFwdCtasPerSm;
    // tcgen05: 64-pixel tiles of four lanes per pixel (eight warps for the read-back), W of at most 128
    // rows and whole 64-wide slabs of at most 128 columns
    const bool tc_shape = g.TH * g.TW == kTcPix && g.G * g.nslice == 4 && Cx % 64 == 0 && Cx <= 128 &&
                          g.P <= kTcRows;
    if (tc_shape && forward_linear_smem_bytes(g, Cx, 2) + 1024 <= budget) return 2;
    return forward_linear_smem_bytes(g, Cx, 1) + 1024 <= budget ? 1 : 0;
}

cudaError_t launch_forward_linear(const Geometry& g, int dtype, const void* value, const void* x, const void* w,
                                  const void* b, void* out, void* om_out, int Cx, cudaStream_t stream) {
    switch (dtype) {
        case 1: {
            const int mode = forward_linear_mode(g, Cx);
            const LinearArgs<__half> lin{static_cast<const __half*>(x), static_cast<const __half*>(w),
                                         static_cast<const __half*>(b), static_cast<__half*>(om_out), Cx,
                                         mode == 1 ? 1 : 0, mode == 2 ? 1 : 0};
            return launch_vec<__half, true>(g, g.vec, value, nullptr, out, lin, stream);
        }
        case 2: {
            const int mode = forward_linear_mode(g, Cx);
            const LinearArgs<__nv_bfloat16> lin{static_cast<const __nv_bfloat16*>(x),
                                                static_cast<const __nv_bfloat16*>(w),
                                                static_cast<const __nv_bfloat16*>(b),
                                                static_cast<__nv_bfloat16*>(om_out), Cx, mode == 1 ? 1 : 0,
                                                mode == 2 ? 1 : 0};
            return launch_vec<__nv_bfloat16, true>(g, g.vec, value, nullptr, out, lin, stream);
        }
        default: return cudaErrorInvalidValue;
    }
}

bool forward_proj_shape_ok(const Geometry& g, int Cout) {
    const int npix = g.pix_per_cta;
    return (npix == 16 || npix == 32 || npix == 64) && g.TH * g.TW == npix && g.C % 64 == 0 && g.C <= 256 &&
           Cout >= 16 && Cout % 16 == 0 && Cout <= kTcRows && samples_threads(g) == npix * g.G * g.nslice;
}

size_t forward_proj_smem_bytes(const Geometry& g, int Cout) {
    return 2 * static_cast<size_t>(g.pix_per_cta) * g.P * 2 + forward_exps_bytes(g) + proj_extra_bytes(g, Cout);
}

cudaError_t launch_forward_proj(const Geometry& g, int dtype, const void* value, const void* om, const void* w,
                                const void* b, void* out, void* core_out, int Cout, cudaStream_t stream) {
    switch (dtype) {
        case 1: {
            LinearArgs<__half> a{};
            a.pw = static_cast<const __half*>(w);
            a.pb = static_cast<const __half*>(b);
            a.core_out = static_cast<__half*>(core_out);
            a.Cout = Cout;
            return launch_vec<__half, false, true>(g, g.vec, value, om, out, a, stream);
        }
        case 2: {
            LinearArgs<__nv_bfloat16> a{};
            a.pw = static_cast<const __nv_bfloat16*>(w);
            a.pb = static_cast<const __nv_bfloat16*>(b);
            a.core_out = static_cast<__nv_bfloat16*>(core_out);
            a.Cout = Cout;
            return launch_vec<__nv_bfloat16, false, true>(g, g.vec, value, om, out, a, stream);
        }
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t forward_tc_status(unsigned* status, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(status, g_fwd_linear_status, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0u;
        e = cudaMemcpyToSymbol(g_fwd_linear_status, &zero, sizeof(unsigned));
    }
    return e;
}

size_t forward_smem_bytes(const Geometry& g, int elem_bytes) {
    return forward_bufs(g, elem_bytes, 0) * static_cast<size_t>(g.pix_per_cta) * g.P * elem_bytes +
           forward_exps_bytes(g);
}

cudaError_t launch_forward(const Geometry& g, int dtype, const void* value, const void* om, void* out,
                           cudaStream_t stream) {
    const int vec = g.vec;
    switch (dtype) {
        case 0: return launch_vec<float>(g, vec, value, om, out, LinearArgs<float>{}, stream);
        case 1: return launch_vec<__half>(g, vec, value, om, out, LinearArgs<__half>{}, stream);
        case 2: return launch_vec<__nv_bfloat16>(g, vec, value, om, out, LinearArgs<__nv_bfloat16>{}, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
