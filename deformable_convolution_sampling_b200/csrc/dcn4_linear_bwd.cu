// dcn4_linear_bwd.cu — backward of the merged offset/mask linear layer.
//
// The DCNv4 module forms offsets and dynamic weights with one linear layer
// (CSDN summary of "Efficient Deformable ConvNets", section 2.2 "DCN模块的微设计"),
// offset_mask = x W^T + b, which dcn4_forward_linear fuses into the forward.
// Its gradients, with g = grad_offset_mask as an [M, P] matrix (M output
// pixels; the padding columns of g are zero):
//     grad_x [M, Cx] = g W          grad_W [P, Cx] = g^T x          grad_b [P] = sum_m g[m, :]
// Both products run on the tensor cores (mma.sync m16n8k16, fp16/bf16 in,
// fp32 accumulation) from tiles staged in shared memory with cp.async.  They
// are bound by HBM (g, x read once, grad_x written once: about 40 FLOP per
// byte, far below the tensor pipe's ridge), so the tiles are sized for
// streaming, not for tensor throughput.
//   grad_x: a CTA per 128 x 64 output tile, the K = P loop in chunks of 32.
//   grad_W: a CTA per 64 x 64 output tile and M chunk (split K), partial sums
//           added into an fp32 accumulator with vector reductions, then one
//           rounding kernel; the CTAs of the first column tile also sum g's
//           columns for grad_b.
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

// ---------------------------------------------------------------------------
// grad_x = g W: A = g [M, P] (row-major, k = p), B = W [P, Cx] (k-major rows).
// ---------------------------------------------------------------------------
constexpr int kXM = 128, kXN = 64, kXK = 32;
constexpr int kXLdA = kXK + 8, kXLdB = kXN + 8;  // padded rows: conflict-free ldmatrix

template <typename T>
__global__ void __launch_bounds__(kLbThreads) linear_grad_x_kernel(const T* __restrict__ g, const T* __restrict__ w,
                                                                   T* __restrict__ gx, long long M, int P, int Cx) {
    __shared__ __align__(16) T a_s[2][kXM][kXLdA];
    __shared__ __align__(16) T b_s[2][kXK][kXLdB];
    const long long m0 = static_cast<long long>(blockIdx.x) * kXM;
    const int n0 = blockIdx.y * kXN;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wm = warp >> 1, wn = warp & 1;  // 4 x 2 warps of 32 x 32
    constexpr int EPV = 8;                    // 16-bit elements per 16-byte chunk

    auto stage = [&](int kc, int buf) {
        const int k0 = kc * kXK;
        // A: 128 rows x 32 columns = 512 chunks
        for (int i = threadIdx.x; i < kXM * (kXK / EPV); i += blockDim.x) {
            const int r = i / (kXK / EPV), c = (i - r * (kXK / EPV)) * EPV;
            const long long m = m0 + r;
            const bool ok = m < M && k0 + c < P;
            cp_async16(&a_s[buf][r][c], g + (ok ? m * P + k0 + c : 0), ok);
        }
        // B: 32 rows x 64 columns = 256 chunks
        for (int i = threadIdx.x; i < kXK * (kXN / EPV); i += blockDim.x) {
            const int r = i / (kXN / EPV), c = (i - r * (kXN / EPV)) * EPV;
            const bool ok = k0 + r < P && n0 + c < Cx;
            cp_async16(&b_s[buf][r][c], w + (ok ? static_cast<long long>(k0 + r) * Cx + n0 + c : 0), ok);
        }
        asm volatile("cp.async.commit_group;");
    };

    float acc[2][4][4] = {};
    const int kchunks = (P + kXK - 1) / kXK;
    stage(0, 0);
    for (int kc = 0; kc < kchunks; ++kc) {
        if (kc + 1 < kchunks) {
            stage(kc + 1, (kc + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int buf = kc & 1;
#pragma unroll
        for (int ks = 0; ks < kXK / 16; ++ks) {
            uint32_t a[2][4], b[4][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
                ldsm_x4(a[mt], &a_s[buf][wm * 32 + mt * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                // two n8 tiles per x4.trans: lanes 0-15 rows k of tile 2np, lanes 16-31 of tile 2np+1
                uint32_t r[4];
                ldsm_x4_t(r, &b_s[buf][ks * 16 + (lane & 15)][wn * 32 + np * 16 + (lane >> 4) * 8]);
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
        __syncthreads();
    }
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = n0 + wn * 32 + nt * 8 + tq * 2;
            if (col >= Cx) continue;
            const long long r0 = m0 + wm * 32 + mt * 16 + gq, r1 = r0 + 8;
            if (r0 < M) *reinterpret_cast<uint32_t*>(gx + r0 * Cx + col) = pack_pair<T>(acc[mt][nt][0], acc[mt][nt][1]);
            if (r1 < M) *reinterpret_cast<uint32_t*>(gx + r1 * Cx + col) = pack_pair<T>(acc[mt][nt][2], acc[mt][nt][3]);
        }
}

// ---------------------------------------------------------------------------
// grad_W += g^T x over one chunk of rows: A = g^T (from g [m][p] with
// ldmatrix.trans), B = x [m][c] (k = m).  grad_b from the column sums of g.
// ---------------------------------------------------------------------------
constexpr int kWP = 64, kWC = 64, kWK = 32;
constexpr int kWLd = 64 + 8;

__device__ __forceinline__ void red_add2(float* dst, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(a), "f"(b) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kLbThreads) linear_grad_w_kernel(const T* __restrict__ g, const T* __restrict__ x,
                                                                   float* __restrict__ wacc, float* __restrict__ bacc,
                                                                   long long M, int P, int Cx, long long mchunk) {
    __shared__ __align__(16) T g_s[2][kWK][kWLd];  // [m][p]
    __shared__ __align__(16) T x_s[2][kWK][kWLd];  // [m][c]
    __shared__ float b_part[kLbThreads];
    const int p0 = blockIdx.x * kWP, c0 = blockIdx.y * kWC;
    const long long mb = static_cast<long long>(blockIdx.z) * mchunk;
    const long long me = std::min<long long>(M, mb + mchunk);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wp = warp >> 2, wc = warp & 3;  // 2 x 4 warps of 32 (p) x 16 (c)
    constexpr int EPV = 8;
    const bool sum_b = bacc != nullptr && blockIdx.y == 0;

    auto stage = [&](long long m, int buf) {
        for (int i = threadIdx.x; i < kWK * (kWP / EPV) * 2; i += blockDim.x) {
            const int half = i / (kWK * (kWP / EPV));  // 0: g, 1: x
            const int j = i - half * (kWK * (kWP / EPV));
            const int r = j / (kWP / EPV), c = (j - r * (kWP / EPV)) * EPV;
            const long long mm = m + r;
            if (half == 0) {
                const bool ok = mm < me && p0 + c < P;
                cp_async16(&g_s[buf][r][c], g + (ok ? mm * P + p0 + c : 0), ok);
            } else {
                const bool ok = mm < me && c0 + c < Cx;
                cp_async16(&x_s[buf][r][c], x + (ok ? mm * Cx + c0 + c : 0), ok);
            }
        }
        asm volatile("cp.async.commit_group;");
    };

    float acc[2][2][4] = {};
    float bsum = 0.f;  // column p0 + (threadIdx.x & 63) of g over this thread's rows
    const int nk = static_cast<int>((me - mb + kWK - 1) / kWK);
    if (nk > 0) stage(mb, 0);
    for (int kc = 0; kc < nk; ++kc) {
        if (kc + 1 < nk) {
            stage(mb + static_cast<long long>(kc + 1) * kWK, (kc + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int buf = kc & 1;
        if (sum_b) {
            // 256 threads: column threadIdx & 63, rows (threadIdx >> 6) + 4j
            for (int r = threadIdx.x >> 6; r < kWK; r += kLbThreads / 64) bsum += to_f32(g_s[buf][r][threadIdx.x & 63]);
        }
#pragma unroll
        for (int ks = 0; ks < kWK / 16; ++ks) {
            uint32_t a[2][4], b[2][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                // A[p][m] = g[m][p]: submatrices (p 0-7, m 0-7), (p 8-15, m 0-7), (p 0-7, m 8-15), (p 8-15, m 8-15)
                const int mrow = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int pcol = wp * 32 + mt * 16 + (((lane >> 3) & 1) << 3);
                ldsm_x4_t(a[mt], &g_s[buf][mrow][pcol]);
            }
            {
                uint32_t r[4];
                ldsm_x4_t(r, &x_s[buf][ks * 16 + (lane & 15)][wc * 16 + (lane >> 4) * 8]);
                b[0][0] = r[0];
                b[0][1] = r[1];
                b[1][0] = r[2];
                b[1][1] = r[3];
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) mma16816<T>(acc[mt][nt], a[mt], b[nt]);
        }
        __syncthreads();
    }
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = c0 + wc * 16 + nt * 8 + tq * 2;
            const int r0 = p0 + wp * 32 + mt * 16 + gq, r1 = r0 + 8;
            if (col >= Cx) continue;
            if (r0 < P) red_add2(wacc + static_cast<long long>(r0) * Cx + col, acc[mt][nt][0], acc[mt][nt][1]);
            if (r1 < P) red_add2(wacc + static_cast<long long>(r1) * Cx + col, acc[mt][nt][2], acc[mt][nt][3]);
        }
    if (sum_b) {
        b_part[threadIdx.x] = bsum;
        __syncthreads();
        if (threadIdx.x < 64 && p0 + static_cast<int>(threadIdx.x) < P) {
            float s = 0.f;
            for (int j = 0; j < kLbThreads / 64; ++j) s += b_part[threadIdx.x + 64 * j];
            atomicAdd(bacc + p0 + threadIdx.x, s);
        }
    }
}

// out[i] = round(acc[i]) for n elements.
template <typename T>
__global__ void linear_round_kernel(const float* __restrict__ acc, T* __restrict__ out, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        out[i] = from_f32<T>(acc[i]);
}

template <typename T>
cudaError_t linear_backward_typed(long long M, int P, int Cx, const void* x, const void* w, const void* gom,
                                  void* gx, void* gw, void* gb, float* ws, cudaStream_t stream) {
    const T* g = static_cast<const T*>(gom);
    if (gx) {
        const dim3 grid(static_cast<unsigned>((M + kXM - 1) / kXM), static_cast<unsigned>((Cx + kXN - 1) / kXN));
        linear_grad_x_kernel<T><<<grid, kLbThreads, 0, stream>>>(g, static_cast<const T*>(w), static_cast<T*>(gx), M, P,
                                                                 Cx);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!gw && !gb) return cudaSuccess;
    const long long wsz = static_cast<long long>(P) * Cx;
    cudaError_t e = cudaMemsetAsync(ws, 0, (wsz + P) * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const int pt = (P + kWP - 1) / kWP, ct = (Cx + kWC - 1) / kWC;
    // split K so that the grid holds about four CTAs per SM
    const long long want = std::max<long long>(1, 600 / (pt * ct));
    long long mchunk = (M + want - 1) / want;
    mchunk = std::max<long long>(256, (mchunk + kWK - 1) / kWK * kWK);
    const long long zc = (M + mchunk - 1) / mchunk;
    const dim3 grid(static_cast<unsigned>(pt), static_cast<unsigned>(ct), static_cast<unsigned>(std::max<long long>(1, zc)));
    linear_grad_w_kernel<T><<<grid, kLbThreads, 0, stream>>>(g, static_cast<const T*>(x), ws, gb ? ws + wsz : nullptr,
                                                             M, P, Cx, mchunk);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (gw) {
        linear_round_kernel<T><<<static_cast<unsigned>(std::min<long long>((wsz + 255) / 256, 4096)), 256, 0, stream>>>(
            ws, static_cast<T*>(gw), wsz);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (gb) {
        linear_round_kernel<T><<<static_cast<unsigned>((P + 255) / 256), 256, 0, stream>>>(ws + wsz, static_cast<T*>(gb), P);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

size_t linear_backward_workspace_bytes(int P, int Cx) {
    return (static_cast<size_t>(P) * Cx + P) * sizeof(float);
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
