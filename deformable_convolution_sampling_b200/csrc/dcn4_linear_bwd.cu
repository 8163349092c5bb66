// dcn4_linear_bwd.cu — backward of the merged offset/mask linear layer.
//
// The DCNv4 module forms offsets and dynamic weights with one linear layer
// (CSDN summary of "Efficient Deformable ConvNets", section 2.2 "DCN模块的微设计"),
// offset_mask = x W^T + b, which dcn4_forward_linear fuses into the forward.
// Its gradients, with g = grad_offset_mask as an [M, P] matrix (M output
// pixels; the padding columns of g are zero):
//     grad_x [M, Cx] = g W          grad_W [P, Cx] = g^T x          grad_b [P] = sum_m g[m, :]
// Both products run on the tensor cores (mma.sync m16n8k16, fp16/bf16 in,
// fp32 accumulation) from tiles staged in shared memory by a cp.async ring.  They are bound by HBM (g and x read, grad_x written: 40-60
// FLOP per byte, far below the tensor pipe's ridge), so the kernels are built
// for streaming: long-lived CTAs whose ring runs across tile boundaries.
//   grad_x: persistent CTAs walk (128 x 64 output tile, 32-deep chunk of P)
//           pairs through a four-deep ring; 32 x 32 warp tiles.
//   grad_W: a CTA per 128 x 64 output tile and range of rows (split K), 32 rows
//           per stage, four-deep ring; 32 x 32 warp tiles.  grad_b rides on the same A
//           fragments: one more MMA per step against a constant B whose first
//           column is ones.  Partial tiles are added into fp32 accumulators
//           with vector reductions; the last CTA to finish rounds them once.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "dcn4_common.cuh"

namespace dcn4 {
namespace {

constexpr int kLbThreads = 256;

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src, bool valid) {
    const unsigned da = static_cast<unsigned>(__cvta_generic_to_shared(dst_smem));
    const int n = valid ? 16 : 0;  // 0 source bytes: the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(da), "l"(src), "r"(n));
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
    const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

// d += a (16x16, row fragments) * b (16x8, column fragments), fp32 accumulation.
template <typename T>
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, const uint32_t* b) {
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
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi) {
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

constexpr int kPad = 8;  // padded smem rows (16 bytes): conflict-free ldmatrix

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Rounds one 128 x 64 tile of the fp32 grad_W accumulator (and, for the first
// column tile, its 128 grad_b entries) into the outputs: every load of a thread
// is issued before the first store.
template <typename T, int NT>
__device__ __forceinline__ void round_tile(const float* wacc, const float* bacc, T* gw, T* gb, int P, int Cx, int p0,
                                           int c0, bool with_b) {
    constexpr int kVec = 128 * 64 / 4 / NT;  // float4 groups per thread
    if (gw) {
        float4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int e = threadIdx.x + u * NT, r = e >> 4, c = (e & 15) * 4;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p0 + r < P && c0 + c < Cx)
                v[u] = __ldcg(reinterpret_cast<const float4*>(wacc + static_cast<long long>(p0 + r) * Cx + c0 + c));
        }
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int e = threadIdx.x + u * NT, r = e >> 4, c = (e & 15) * 4;
            if (p0 + r < P && c0 + c < Cx)
                *reinterpret_cast<uint2*>(gw + static_cast<long long>(p0 + r) * Cx + c0 + c) =
                    make_uint2(pack_pair<T>(v[u].x, v[u].y), pack_pair<T>(v[u].z, v[u].w));
        }
    }
    if (gb && with_b)
        for (int r = threadIdx.x; r < 128; r += NT)
            if (p0 + r < P) gb[p0 + r] = from_f32<T>(__ldcg(bacc + p0 + r));
}

// ---------------------------------------------------------------------------
// grad_x = g W: A = g [M, P] (row-major, k = p), B = W [P, Cx] (k-major rows).
// ---------------------------------------------------------------------------
constexpr int kXM = 128, kXN = 64, kXK = 32, kXStages = 4;
template <typename T>
struct XStage {
    T a[kXM][kXK + kPad];
    T b[kXK][kXN + kPad];
};

template <typename T>
__global__ void __launch_bounds__(kLbThreads, 3)
    linear_grad_x_kernel(const T* __restrict__ g, const T* __restrict__ w, T* __restrict__ gx, long long M, int P,
                         int Cx, long long ntiles, int ntiles_n, int nk) {
    extern __shared__ __align__(16) unsigned char lin_smem[];
    XStage<T>* st = reinterpret_cast<XStage<T>*>(lin_smem);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wm = warp >> 1, wn = warp & 1;  // 4 x 2 warps of 32 x 32
    constexpr int EPV = 8;                    // 16-bit elements per 16-byte chunk
    if (static_cast<long long>(blockIdx.x) >= ntiles) return;
    // this thread's 16-byte chunks: A rows ar and ar + 64 at column ac; B row br at column bc
    const int ar = threadIdx.x / (kXK / EPV), ac = (threadIdx.x % (kXK / EPV)) * EPV;
    const int br = threadIdx.x / (kXN / EPV), bc = (threadIdx.x % (kXN / EPV)) * EPV;
    static_assert(kXM * (kXK / EPV) == 2 * kLbThreads && kXK * (kXN / EPV) == kLbThreads, "chunk split");

    // (tile, chunk) walk of the loads, kXStages - 1 ahead of the compute walk
    long long ld_tile = blockIdx.x;
    int ld_kc = 0;
    auto load = [&](int slot) {
        const long long tm = ld_tile / ntiles_n;
        const int n0 = static_cast<int>(ld_tile - tm * ntiles_n) * kXN;
        const long long m0 = tm * kXM;
        const int k0 = ld_kc * kXK;
        XStage<T>& s = st[slot];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = ar + (kXM / 2) * i;
            const long long m = m0 + r;
            const bool ok = m < M && k0 + ac < P;
            cp_async16(&s.a[r][ac], g + (ok ? m * P + k0 + ac : 0), ok);
        }
        const bool okb = k0 + br < P && n0 + bc < Cx;
        cp_async16(&s.b[br][bc], w + (okb ? static_cast<long long>(k0 + br) * Cx + n0 + bc : 0), okb);
        if (++ld_kc == nk) {
            ld_kc = 0;
            ld_tile += gridDim.x;
        }
    };

    float acc[2][4][4] = {};
    for (int j = 0; j < kXStages - 1; ++j) {
        if (ld_tile < ntiles) load(j);
        cp_async_commit();
    }
    long long tile = blockIdx.x;
    int kc = 0, slot = 0;
    while (tile < ntiles) {
        cp_async_wait<kXStages - 2>();
        __syncthreads();  // this slot landed for every thread; the slot used last is free again
        if (ld_tile < ntiles) load(slot == 0 ? kXStages - 1 : slot - 1);
        cp_async_commit();
        const XStage<T>& s = st[slot];
#pragma unroll
        for (int ks = 0; ks < kXK / 16; ++ks) {
            uint32_t a[2][4], b[4][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
                ldsm_x4(a[mt], &s.a[wm * 32 + mt * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                // two n8 tiles per x4.trans: lanes 0-15 address the k rows of tile 2np, lanes 16-31 of 2np+1
                uint32_t r[4];
                ldsm_x4_t(r, &s.b[ks * 16 + (lane & 15)][wn * 32 + np * 16 + (lane >> 4) * 8]);
                b[2 * np][0] = r[0];
                b[2 * np][1] = r[1];
                b[2 * np + 1][0] = r[2];
                b[2 * np + 1][1] = r[3];
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mma16816<T>(acc[mt][nt], a[mt], b[nt]);
        }
        slot = slot + 1 == kXStages ? 0 : slot + 1;
        if (++kc == nk) {  // last chunk of this tile: round once and store
            const long long tm = tile / ntiles_n;
            const int n0 = static_cast<int>(tile - tm * ntiles_n) * kXN;
            const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int col = n0 + wn * 32 + nt * 8 + tq * 2;
                    const long long r0 = tm * kXM + wm * 32 + mt * 16 + gq, r1 = r0 + 8;
                    if (col < Cx) {
                        if (r0 < M)
                            *reinterpret_cast<uint32_t*>(gx + r0 * Cx + col) = pack_pair<T>(acc[mt][nt][0], acc[mt][nt][1]);
                        if (r1 < M)
                            *reinterpret_cast<uint32_t*>(gx + r1 * Cx + col) = pack_pair<T>(acc[mt][nt][2], acc[mt][nt][3]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
                }
            kc = 0;
            tile += gridDim.x;
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// grad_W += g^T x over a range of rows: A = g^T (from g [m][p] with
// ldmatrix.trans), B = x [m][c] (k = m).  grad_b from the same A fragments.
// ---------------------------------------------------------------------------
constexpr int kWP = 128, kWC = 64, kWK = 32, kWStages = 4;
template <typename T>
struct WStage {
    T g[kWK][kWP + kPad];  // [m][p]
    T x[kWK][kWC + kPad];  // [m][c]
};

__device__ __forceinline__ void red_add2(float* dst, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(a), "f"(b) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kLbThreads, 3)
    linear_grad_w_kernel(const T* __restrict__ g, const T* __restrict__ x, float* __restrict__ wacc,
                         float* __restrict__ bacc, unsigned* __restrict__ done, T* __restrict__ gw,
                         T* __restrict__ gb, long long M, int P, int Cx, int ntile, int ct, long long mchunk) {
    extern __shared__ __align__(16) unsigned char lin_smem[];
    WStage<T>* st = reinterpret_cast<WStage<T>*>(lin_smem);
    __shared__ unsigned ticket;
    const int tile = blockIdx.x % ntile;  // ntile = (P tiles) x (Cx tiles); blocks of one split run together
    const long long split = blockIdx.x / ntile;
    const int tp = tile / ct, tc = tile - tp * ct;
    const int p0 = tp * kWP, c0 = tc * kWC;
    const long long mb = split * mchunk;
    const long long me = std::min<long long>(M, mb + mchunk);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wp = warp >> 1, wc = warp & 1;  // 4 x 2 warps of 32 (p) x 32 (c)
    constexpr int EPV = 8;
    const bool sum_b = bacc != nullptr && tc == 0 && wc == 0;
    const int nk = static_cast<int>((me - mb + kWK - 1) / kWK);
    // this thread's 16-byte chunks: g rows gr and gr + 16 at column gc; x row xr at column xc
    const int gr = threadIdx.x / (kWP / EPV), gc = (threadIdx.x % (kWP / EPV)) * EPV;
    const int xr = threadIdx.x / (kWC / EPV), xc = (threadIdx.x % (kWC / EPV)) * EPV;
    static_assert(kWK * (kWP / EPV) == 2 * kLbThreads && kWK * (kWC / EPV) == kLbThreads, "chunk split");
    const bool gcol_ok = p0 + gc < P, xcol_ok = c0 + xc < Cx;

    auto load = [&](int j, int slot) {
        const long long m = mb + static_cast<long long>(j) * kWK;
        WStage<T>& s = st[slot];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = gr + (kWK / 2) * i;
            const long long mm = m + r;
            const bool ok = mm < me && gcol_ok;
            cp_async16(&s.g[r][gc], g + (ok ? mm * P + p0 + gc : 0), ok);
        }
        const long long mm = m + xr;
        const bool ok = mm < me && xcol_ok;
        cp_async16(&s.x[xr][xc], x + (ok ? mm * Cx + c0 + xc : 0), ok);
    };

    // B operand whose first column is ones: A * ones_b puts the row sums of A in column 0
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t one2 = gq == 0 ? pack_pair<T>(1.f, 1.f) : 0u;
    const uint32_t ones_b[2] = {one2, one2};

    float acc[2][4][4] = {};
    float accb[2][4] = {};
    for (int j = 0; j < kWStages - 1; ++j) {
        if (j < nk) load(j, j);
        cp_async_commit();
    }
    int slot = 0;
    for (int j = 0; j < nk; ++j) {
        cp_async_wait<kWStages - 2>();
        __syncthreads();
        if (j + kWStages - 1 < nk) load(j + kWStages - 1, slot == 0 ? kWStages - 1 : slot - 1);
        cp_async_commit();
        const WStage<T>& s = st[slot];
        slot = slot + 1 == kWStages ? 0 : slot + 1;
#pragma unroll
        for (int ks = 0; ks < kWK / 16; ++ks) {
            uint32_t a[2][4], b[4][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                // A[p][m] = g[m][p]: submatrices (p 0-7, m 0-7), (p 8-15, m 0-7), (p 0-7, m 8-15), (p 8-15, m 8-15)
                const int mrow = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int pcol = wp * 32 + mt * 16 + (((lane >> 3) & 1) << 3);
                ldsm_x4_t(a[mt], &s.g[mrow][pcol]);
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t r[4];
                ldsm_x4_t(r, &s.x[ks * 16 + (lane & 15)][wc * 32 + np * 16 + (lane >> 4) * 8]);
                b[2 * np][0] = r[0];
                b[2 * np][1] = r[1];
                b[2 * np + 1][0] = r[2];
                b[2 * np + 1][1] = r[3];
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mma16816<T>(acc[mt][nt], a[mt], b[nt]);
                if (sum_b) mma16816<T>(accb[mt], a[mt], ones_b);
            }
        }
    }
    cp_async_wait<0>();

#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const int r0 = p0 + wp * 32 + mt * 16 + gq, r1 = r0 + 8;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = c0 + wc * 32 + nt * 8 + tq * 2;
            if (col >= Cx) continue;
            if (r0 < P) red_add2(wacc + static_cast<long long>(r0) * Cx + col, acc[mt][nt][0], acc[mt][nt][1]);
            if (r1 < P) red_add2(wacc + static_cast<long long>(r1) * Cx + col, acc[mt][nt][2], acc[mt][nt][3]);
        }
        if (sum_b && tq == 0) {  // column 0 of the ones product: rows r0 and r1
            if (r0 < P) atomicAdd(bacc + r0, accb[mt][0]);
            if (r1 < P) atomicAdd(bacc + r1, accb[mt][2]);
        }
    }

    // The last CTA of this output tile rounds it once (its fence orders the other
    // CTAs' reductions, which precede their tickets, before its reads).
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) ticket = atomicAdd(done + tile, 1u);
    __syncthreads();
    if (ticket != gridDim.x / ntile - 1) return;
    __threadfence();
    round_tile<T, kLbThreads>(wacc, bacc, gw, gb, P, Cx, p0, c0, tc == 0);
}

// ---------------------------------------------------------------------------
// grad_x = g W on the fifth-generation tensor cores (tcgen05).  One thread
// issues the MMAs (M = 128 rows of g, N = 64 columns of grad_x, K = 16 each),
// operands read from shared memory by descriptor, the fp32 accumulator in
// tensor memory; the CTA's 128 threads stage the operands and read the
// accumulator back.  Operands use the no-swizzle canonical layouts, 8 x 8
// core matrices of 128 bytes (8 rows of 16 bytes):
//   A = g  (K-major): element (m, k) at (m/8)*512 + (k/8)*128 + (m%8)*16 + (k%8)*2
//   B = W  (N-major): element (k, n) at (k/8)*1024 + (n/8)*128 + (k%8)*16 + (n%8)*2
// The ring has kTStages slots of 32 rows of K, loaded kTDepth ahead: a slot is
// refilled two iterations after the MMAs that read it were issued, so the
// loads never wait on the tensor cores' latency.
// ---------------------------------------------------------------------------
constexpr int kTM = 128, kTN = 64, kTK = 32, kTStages = 6, kTDepth = 4, kTThreads = 128;
constexpr int kTABytes = kTM * kTK * 2;               // 8 KB
constexpr int kTBBytes = kTK * kTN * 2;               // 4 KB
constexpr int kTStageBytes = kTABytes + kTBBytes;     // 12 KB
constexpr int kTSlack = 16 * 1024;                    // guard band after the ring
constexpr int kTSmem = kTStages * kTStageBytes + kTSlack;
constexpr int kTWaitSpins = 1 << 22;                  // bound of every mbarrier wait
constexpr unsigned kLinStatusTimeout = 1u;            // a wait gave up (status word)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16_s(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets (all in 16-byte units), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16 with fp32 accumulation: operand format
// (0 fp16, 1 bf16) for A and B, their majorness (0 K, 1 M/N), N / 8 and M / 16.
template <typename T>
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, int a_mn, int b_mn) {
    const uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum ? 1 : 0));
}

__device__ __forceinline__ void umma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Waits (bounded) for the completion of the phase of parity `parity`; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    for (int i = 0; i < kTWaitSpins; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, P1;\n\t}"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <typename T>
__global__ void __launch_bounds__(kTThreads, 2)
    linear_grad_x_tc_kernel(const T* __restrict__ g, const T* __restrict__ w, T* __restrict__ gx, long long M, int P,
                            int Cx, long long ntiles, int ntiles_n, int nk, unsigned* __restrict__ status) {
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    __shared__ __align__(8) uint64_t mbar[kTStages];
    __shared__ uint32_t taddr_s;
    if (static_cast<long long>(blockIdx.x) >= ntiles) return;  // whole CTA, before anything is held
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t ring = smem_u32(tc_smem);
    if (tid == 0) {
        for (int s = 0; s < kTStages; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar[s])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // 64 fp32 columns x 128 lanes of tensor memory: the accumulator
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&taddr_s)),
                     "r"(kTN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = taddr_s;
    constexpr uint32_t idesc = umma_idesc<T>(kTM, kTN, 0, 1);

    // (tile, chunk) walk of the loads, kTStages - 1 ahead of the MMAs
    long long ld_tile = blockIdx.x;
    int ld_kc = 0;
    auto load = [&](int slot) {
        const long long tm = ld_tile / ntiles_n;
        const int n0 = static_cast<int>(ld_tile - tm * ntiles_n) * kTN;
        const long long m0 = tm * kTM;
        const int k0 = ld_kc * kTK;
        const uint32_t sa = ring + slot * kTStageBytes, sb = sa + kTABytes;
#pragma unroll
        for (int u = 0; u < kTM * (kTK / 8) / kTThreads; ++u) {  // A: 128 rows x 4 chunks of 16 bytes
            const int i = tid + u * kTThreads, m = i >> 2, kg = i & 3;
            const bool ok = m0 + m < M && k0 + kg * 8 < P;
            cp_async16_s(sa + (m >> 3) * 512 + kg * 128 + (m & 7) * 16, g + (ok ? (m0 + m) * P + k0 + kg * 8 : 0), ok);
        }
#pragma unroll
        for (int u = 0; u < kTK * (kTN / 8) / kTThreads; ++u) {  // B: 32 rows x 8 chunks
            const int i = tid + u * kTThreads, k = i >> 3, ng = i & 7;
            const bool ok = k0 + k < P && n0 + ng * 8 < Cx;
            cp_async16_s(sb + (k >> 3) * 1024 + ng * 128 + (k & 7) * 16,
                         w + (ok ? static_cast<long long>(k0 + k) * Cx + n0 + ng * 8 : 0), ok);
        }
        if (++ld_kc == nk) {
            ld_kc = 0;
            ld_tile += gridDim.x;
        }
    };

    uint32_t phase = 0, pending = 0;  // per slot: parity of its next completion; a commit not yet waited for
    int aborted = 0;                  // this thread gave up a wait; the CTA stops at the next barrier
    auto wait_slot = [&](int s) {
        if (!((pending >> s) & 1u)) return;
        if (!mbar_wait(smem_u32(&mbar[s]), (phase >> s) & 1u)) aborted = 1;
        phase ^= 1u << s;
        pending &= ~(1u << s);
    };

    for (int j = 0; j < kTDepth; ++j) {
        if (ld_tile < ntiles) load(j);
        cp_async_commit();
    }
    long long tile = blockIdx.x;
    int kc = 0, slot = 0, ld_slot = kTDepth;
    while (tile < ntiles) {
        wait_slot(ld_slot);  // the MMAs that last read ld_slot (two iterations ago) are done
        if (ld_tile < ntiles) load(ld_slot);
        cp_async_commit();
        ld_slot = ld_slot + 1 == kTStages ? 0 : ld_slot + 1;
        cp_async_wait<kTDepth>();                   // this thread's copies of `slot` landed
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // ... and are visible to the tensor cores
        if (__syncthreads_or(aborted)) break;
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sa = ring + slot * kTStageBytes, sb = sa + kTABytes;
#pragma unroll
            for (int q = 0; q < kTK / 16; ++q)  // K = 16 per MMA: two core matrices of A, two rows of B's
                umma_f16(tmem, umma_desc(sa + q * 256, 128, 512), umma_desc(sb + q * 2048, 1024, 128), idesc,
                         kc > 0 || q > 0);
            umma_commit(smem_u32(&mbar[slot]));
        }
        pending |= 1u << slot;
        const int done_slot = slot;
        slot = slot + 1 == kTStages ? 0 : slot + 1;
        if (++kc == nk) {  // the tile's accumulator is complete: read it back, round once, store
            wait_slot(done_slot);
            tc_fence_after();
            const long long tm = tile / ntiles_n;
            const int n0 = static_cast<int>(tile - tm * ntiles_n) * kTN;
            const long long row = tm * kTM + warp * 32 + lane;
            const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
            for (int h = 0; h < kTN / 32; ++h) {
                uint32_t r[32];
                tmem_ld32(lane_addr + h * 32, r);
                if (row < M && !aborted) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int col = n0 + h * 32 + v * 8;
                        if (col >= Cx) continue;
                        uint4 o;
                        o.x = pack_pair<T>(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                        o.y = pack_pair<T>(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                        o.z = pack_pair<T>(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                        o.w = pack_pair<T>(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                        *reinterpret_cast<uint4*>(gx + row * Cx + col) = o;
                    }
                }
            }
            tc_fence_before();  // the next tile's first MMA overwrites the accumulator after the next barrier
            kc = 0;
            tile += gridDim.x;
        }
    }
    cp_async_wait<0>();
    for (int s = 0; s < kTStages; ++s) wait_slot(s);  // no MMA may still read shared or tensor memory
    if (aborted) atomicOr(status, kLinStatusTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTN));
}

// ---------------------------------------------------------------------------
// grad_W += g^T x and grad_b on tcgen05 over one range of rows (split K):
// D [128 rows of W^T's rows p, 80 columns] in tensor memory, K = rows m of g
// and x, 64 per stage.  A = g^T is M-major straight from g's rows (p
// contiguous); B = x is N-major (c contiguous) with two extra column groups
// set once: column 64 all ones, 65-79 zero, so D's column 64 sums g's columns
// (grad_b) with the same MMAs.
//   A: element (p, m) at (m/8)*2048 + (p/8)*128 + (m%8)*16 + (p%8)*2
//   B: element (m, c) at (m/8)*1280 + (c/8)*128 + (m%8)*16 + (c%8)*2
// Ring of kUStages slots of 32 rows, loaded kUDepth ahead (as for grad_x).
// ---------------------------------------------------------------------------
constexpr int kUM = 128, kUN = 64, kUNB = 80, kUK = 32, kUStages = 6, kUDepth = 4;
constexpr int kUABytes = kUK * kUM * 2;               // 8 KB
constexpr int kUBBytes = kUK * kUNB * 2;              // 5 KB
constexpr int kUStageBytes = kUABytes + kUBBytes;     // 13 KB
constexpr int kUSlack = 24 * 1024;
constexpr int kUSmem = kUStages * kUStageBytes + kUSlack;
constexpr int kUTmemCols = 128;                       // 80 used

__device__ __forceinline__ void red_add4(float* dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kTThreads, 2)
    linear_grad_w_tc_kernel(const T* __restrict__ g, const T* __restrict__ x, float* __restrict__ wacc,
                            float* __restrict__ bacc, unsigned* __restrict__ done, unsigned* __restrict__ status,
                            T* __restrict__ gw, T* __restrict__ gb, long long M, int P, int Cx, int ntile, int ct,
                            long long mchunk) {
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    __shared__ __align__(8) uint64_t mbar[kUStages];
    __shared__ uint32_t taddr_s;
    __shared__ unsigned ticket;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x % ntile;  // blocks of one split (the same rows) run together
    const long long split = blockIdx.x / ntile;
    const int tp = tile / ct, tc = tile - tp * ct;
    const int p0 = tp * kUM, c0 = tc * kUN;
    const long long mb = split * mchunk;
    const long long me = std::min<long long>(M, mb + mchunk);
    const int nk = static_cast<int>((me - mb + kUK - 1) / kUK);
    const uint32_t ring = smem_u32(tc_smem);
    if (tid == 0) {
        for (int s = 0; s < kUStages; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar[s])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&taddr_s)),
                     "r"(kUTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // the constant column groups of B (8: ones in column 64, 9: zeros), in every stage
    for (int i = tid; i < kUStages * kUK * 2; i += kTThreads) {
        const int s = i / (kUK * 2), r = i - s * (kUK * 2), m = r >> 1, grp = 8 + (r & 1);
        unsigned char* dst = tc_smem + s * kUStageBytes + kUABytes + (m >> 3) * 1280 + grp * 128 + (m & 7) * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (grp == 8) v.x = pack_pair<T>(1.f, 0.f);
        *reinterpret_cast<uint4*>(dst) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = taddr_s;
    constexpr uint32_t idesc = umma_idesc<T>(kUM, kUNB, 1, 1);

    auto load = [&](int j, int slot) {
        const long long m = mb + static_cast<long long>(j) * kUK;
        const uint32_t sa = ring + slot * kUStageBytes, sb = sa + kUABytes;
#pragma unroll
        for (int u = 0; u < kUK * (kUM / 8) / kTThreads; ++u) {  // g rows: 32 x 16 chunks of 8 p
            const int i = tid + u * kTThreads, r = i >> 4, pg = i & 15;
            const bool ok = m + r < me && p0 + pg * 8 < P;
            cp_async16_s(sa + (r >> 3) * 2048 + pg * 128 + (r & 7) * 16, g + (ok ? (m + r) * P + p0 + pg * 8 : 0), ok);
        }
#pragma unroll
        for (int u = 0; u < kUK * (kUN / 8) / kTThreads; ++u) {  // x rows: 32 x 8 chunks of 8 c
            const int i = tid + u * kTThreads, r = i >> 3, cg = i & 7;
            const bool ok = m + r < me && c0 + cg * 8 < Cx;
            cp_async16_s(sb + (r >> 3) * 1280 + cg * 128 + (r & 7) * 16, x + (ok ? (m + r) * Cx + c0 + cg * 8 : 0), ok);
        }
    };

    uint32_t phase = 0, pending = 0;
    int aborted = 0;
    auto wait_slot = [&](int s) {
        if (!((pending >> s) & 1u)) return;
        if (!mbar_wait(smem_u32(&mbar[s]), (phase >> s) & 1u)) aborted = 1;
        phase ^= 1u << s;
        pending &= ~(1u << s);
    };
    for (int j = 0; j < kUDepth; ++j) {
        if (j < nk) load(j, j);
        cp_async_commit();
    }
    int slot = 0, ld_slot = kUDepth, last_slot = -1;
    for (int j = 0; j < nk; ++j) {
        wait_slot(ld_slot);  // the MMAs that last read ld_slot (two iterations ago) are done
        if (j + kUDepth < nk) load(j + kUDepth, ld_slot);
        cp_async_commit();
        ld_slot = ld_slot + 1 == kUStages ? 0 : ld_slot + 1;
        cp_async_wait<kUDepth>();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (__syncthreads_or(aborted)) break;
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sa = ring + slot * kUStageBytes, sb = sa + kUABytes;
#pragma unroll
            for (int q = 0; q < kUK / 16; ++q)  // K = 16 rows per MMA: two row groups of A and of B
                umma_f16(tmem, umma_desc(sa + q * 4096, 2048, 128), umma_desc(sb + q * 2560, 1280, 128), idesc,
                         j > 0 || q > 0);
            umma_commit(smem_u32(&mbar[slot]));
        }
        pending |= 1u << slot;
        last_slot = slot;
        slot = slot + 1 == kUStages ? 0 : slot + 1;
    }
    cp_async_wait<0>();
    if (last_slot >= 0) wait_slot(last_slot);
    for (int s = 0; s < kUStages; ++s) wait_slot(s);
    tc_fence_after();

    // Partial tile out: thread = row p of this tile (TMEM lane), 64 columns of
    // grad_W and column 64 (grad_b), added into the fp32 accumulators.
    const int p = p0 + warp * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool live = nk > 0 && !aborted;
#pragma unroll
    for (int h = 0; h < kUN / 32; ++h) {
        uint32_t r[32];
        tmem_ld32(lane_addr + h * 32, r);
        if (live && p < P) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int col = c0 + h * 32 + v * 4;
                if (col < Cx)
                    red_add4(wacc + static_cast<long long>(p) * Cx + col, __uint_as_float(r[4 * v]),
                             __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            }
        }
    }
    {
        uint32_t r[32];
        tmem_ld32(lane_addr + kUN, r);  // columns 64-95: 64 is the ones column
        if (live && p < P && bacc != nullptr && tc == 0) atomicAdd(bacc + p, __uint_as_float(r[0]));
    }
    if (aborted) atomicOr(status, kLinStatusTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols));

    // The last CTA of this output tile rounds it once (its fence orders the other
    // CTAs' reductions, which precede their tickets, before its reads).
    __threadfence();
    __syncthreads();
    if (tid == 0) ticket = atomicAdd(done + tile, 1u);
    __syncthreads();
    if (ticket != gridDim.x / ntile - 1) return;
    __threadfence();
    round_tile<T, kTThreads>(wacc, bacc, gw, gb, P, Cx, p0, c0, tc == 0);
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms > 0 ? sms : 148;
}

constexpr bool kTcgen05 = false;  // tcgen05 products (else mma.sync)

template <typename T>
cudaError_t linear_backward_typed(long long M, int P, int Cx, const void* x, const void* w, const void* gom,
                                  void* gx, void* gw, void* gb, float* ws, cudaStream_t stream) {
    const T* g = static_cast<const T*>(gom);
    const int sms = device_sms();
    const long long wsz = static_cast<long long>(P) * Cx;
    float* wacc = ws;
    float* bacc = ws + wsz;
    unsigned* status = reinterpret_cast<unsigned*>(ws + wsz + P);
    unsigned* done = status + 1;  // one finishing counter per 128 x 64 tile of grad_W
    const long long ntile = static_cast<long long>((P + 127) / 128) * ((Cx + 63) / 64);
    // accumulators, the status word and the finishing counters
    cudaError_t e = cudaMemsetAsync(ws, 0, (wsz + P + 1 + ntile) * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (gx) {
        if constexpr (kTcgen05) {
            e = cudaFuncSetAttribute(linear_grad_x_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTSmem);
            if (e != cudaSuccess) return e;
            const int ntiles_n = (Cx + kTN - 1) / kTN;
            const long long ntiles = (M + kTM - 1) / kTM * ntiles_n;
            const int nk = (P + kTK - 1) / kTK;
            const long long grid = std::min<long long>(ntiles, 2LL * sms);
            linear_grad_x_tc_kernel<T><<<static_cast<unsigned>(grid), kTThreads, kTSmem, stream>>>(
                g, static_cast<const T*>(w), static_cast<T*>(gx), M, P, Cx, ntiles, ntiles_n, nk, status);
        } else {
            const size_t smem = kXStages * sizeof(XStage<T>);
            e = cudaFuncSetAttribute(linear_grad_x_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
            if (e != cudaSuccess) return e;
            const int ntiles_n = (Cx + kXN - 1) / kXN;
            const long long ntiles = (M + kXM - 1) / kXM * ntiles_n;
            const int nk = (P + kXK - 1) / kXK;
            const long long grid = std::min<long long>(ntiles, 3LL * sms);
            linear_grad_x_kernel<T><<<static_cast<unsigned>(grid), kLbThreads, smem, stream>>>(
                g, static_cast<const T*>(w), static_cast<T*>(gx), M, P, Cx, ntiles, ntiles_n, nk);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!gw && !gb) return cudaSuccess;
    const int pt = (P + 127) / 128, ct = (Cx + 63) / 64;
    const int rows = kTcgen05 ? kUK : kWK;
    const int per_sm = kTcgen05 ? 2 : 3;
    // split the rows so that the grid holds about per_sm CTAs per SM, at least a few stages each
    const long long want = std::max<long long>(1, (per_sm * static_cast<long long>(sms) + pt * ct - 1) / (pt * ct));
    long long mchunk = (M + want - 1) / want;
    mchunk = std::max<long long>(4LL * rows, (mchunk + rows - 1) / rows * rows);
    if (mchunk / rows >= 0x7fffffffLL) return cudaErrorInvalidValue;  // stages per CTA must fit an int
    const long long splits = (M + mchunk - 1) / mchunk;
    const long long grid = splits * pt * ct;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if constexpr (kTcgen05) {
        e = cudaFuncSetAttribute(linear_grad_w_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kUSmem);
        if (e != cudaSuccess) return e;
        linear_grad_w_tc_kernel<T><<<static_cast<unsigned>(grid), kTThreads, kUSmem, stream>>>(
            g, static_cast<const T*>(x), wacc, gb ? bacc : nullptr, done, status, static_cast<T*>(gw),
            static_cast<T*>(gb), M, P, Cx, pt * ct, ct, mchunk);
    } else {
        const size_t smem = kWStages * sizeof(WStage<T>);
        e = cudaFuncSetAttribute(linear_grad_w_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        linear_grad_w_kernel<T><<<static_cast<unsigned>(grid), kLbThreads, smem, stream>>>(
            g, static_cast<const T*>(x), wacc, gb ? bacc : nullptr, done, static_cast<T*>(gw), static_cast<T*>(gb), M,
            P, Cx, pt * ct, ct, mchunk);
    }
    return cudaGetLastError();
}

}  // namespace

size_t linear_backward_workspace_bytes(int P, int Cx) {
    // grad_W and grad_b accumulators, the status word, one finishing counter per 128 x 64 tile
    const size_t ntile = static_cast<size_t>((P + 127) / 128) * ((Cx + 63) / 64);
    return (static_cast<size_t>(P) * Cx + P + 1 + ntile) * sizeof(float);
}

cudaError_t launch_linear_backward(int dtype, long long M, int P, int Cx, const void* x, const void* w,
                                   const void* gom, void* gx, void* gw, void* gb, float* ws, cudaStream_t stream) {
    switch (dtype) {
        case 1: return linear_backward_typed<__half>(M, P, Cx, x, w, gom, gx, gw, gb, ws, stream);
        case 2: return linear_backward_typed<__nv_bfloat16>(M, P, Cx, x, w, gom, gx, gw, gb, ws, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn4
