// dcn4_linear_bwd.cu — backward of the merged offset/mask linear layer.
//
// The DCNv4 module forms offsets and dynamic weights with one linear layer
// (CSDN summary of "Efficient Deformable ConvNets", section 2.2 "DCN模块的微设计"),
// offset_mask = x W^T + b, which dcn4_forward_linear fuses into the forward.
// Its gradients, with g = grad_offset_mask as an [M, P] matrix (M output
// pixels; the padding columns of g are zero):
//     grad_x [M, Cx] = g W          grad_W [P, Cx] = g^T x          grad_b [P] = sum_m g[m, :]
// Both products run on the fifth-generation tensor cores (tcgen05.mma,
// fp16/bf16 operands read from shared memory by descriptor, fp32 accumulators
// in tensor memory), fed by TMA in the 128-byte swizzled layout.  Each kernel
// is warp-specialised: a TMA warp fills a ring of stages, an MMA warp consumes
// them, four warps drain the accumulator.  The products are bound by HBM (g
// and x read, grad_x written: 40-60 FLOP per byte, far below the tensor pipe's
// ridge), so the ring is sized for bytes in flight, not for tensor throughput.
//   grad_x: persistent CTAs walk 128 x 64 tiles of grad_x; the accumulator is
//           double-buffered in tensor memory, so one tile's epilogue overlaps
//           the next tile's MMAs.
//   grad_W: a CTA per 128 x 64 tile of grad_W and range of rows (split K);
//           grad_b rides on the same MMAs through a constant ones column of B.
//           Partial tiles are added into fp32 accumulators with vector
//           reductions; the last CTA of each tile rounds it once.
#include <cuda.h>  // tensor-map types (the encoder is resolved at run time)

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "dcn4_common.cuh"
#include "dcn4_tcgen05.cuh"

namespace dcn4 {
namespace {

using namespace tc;

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

// Rounds one 128 x 64 tile of the fp32 grad_W accumulator (and, for the first
// column tile, its 128 grad_b entries) into the outputs: every load of a thread
// is issued before the first store.
template <typename T, int NT>
__device__ __forceinline__ void round_tile(const float* wacc, const float* bacc, T* gw, T* gb, int P, int Cx, int p0,
                                           int c0, bool with_b) {
    constexpr int kGroups = 128 * 64 / 4, kVec = (kGroups + NT - 1) / NT;  // float4 groups: per tile, per thread
    if (gw) {
        float4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int e = threadIdx.x + u * NT, r = e >> 4, c = (e & 15) * 4;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < kGroups && p0 + r < P && c0 + c < Cx)
                v[u] = __ldcg(reinterpret_cast<const float4*>(wacc + static_cast<long long>(p0 + r) * Cx + c0 + c));
        }
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int e = threadIdx.x + u * NT, r = e >> 4, c = (e & 15) * 4;
            if (e < kGroups && p0 + r < P && c0 + c < Cx)
                *reinterpret_cast<uint2*>(gw + static_cast<long long>(p0 + r) * Cx + c0 + c) =
                    make_uint2(pack_pair<T>(v[u].x, v[u].y), pack_pair<T>(v[u].z, v[u].w));
        }
    }
    if (gb && with_b)
        for (int r = threadIdx.x; r < 128; r += NT)
            if (p0 + r < P) gb[p0 + r] = from_f32<T>(__ldcg(bacc + p0 + r));
}

constexpr int kTM = 128, kTN = 64;  // grad_x tile: 128 rows of g x 64 columns
constexpr unsigned kLinStatusTimeout = 1u;  // a wait gave up (status word)
// ---------------------------------------------------------------------------
// tcgen05 products fed by TMA, warp-specialised.  Warp 4 (one lane) loads the
// stages with TMA, warp 5 (one lane) issues the MMAs, warps 0-3 read the
// accumulator back (warp w owns TMEM lanes 32w..32w+31).  Operands use the
// 128-byte swizzled layout: a TMA box 64 elements (128 bytes) wide with
// SWIZZLE_128B lands rows of 128 bytes whose 16-byte chunks are permuted by the
// row index within each 8-row, 1024-byte atom -- the permutation the
// descriptor's SWIZZLE_128B mode undoes.  (Boxes 16 bytes wide in the
// no-swizzle layout were tried first: every row became its own 16-byte
// request, and grad_x took 51 us instead of 19.)
//   K-major operand, 64-wide K slab:  row r at r*128, SBO 1024 (8 rows); the
//       16-wide K step of an MMA moves the start address by 32 bytes.
//   M/N-major operand, 64-wide M/N block: K row k at k*128, SBO 1024 (8 K rows),
//       LBO = distance between 64-wide blocks; the MMA's K step moves 2048 bytes.
// Full / empty barriers per stage, full / empty barriers per accumulator; every
// wait is bounded and gives up at once when another role has given up.
// ---------------------------------------------------------------------------
constexpr int kQThreads = 192;  // 4 epilogue warps, the TMA warp, the MMA warp
constexpr int kQProducer = 4, kQMma = 5;

__device__ __forceinline__ void red_add4(float* dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

constexpr int kUM = 128, kUN = 64, kUTmemCols = 128;  // grad_W tile: 128 rows of W x 64 columns (80 with grad_b)

// grad_x = g W: persistent CTAs walk 128 x 64 tiles of grad_x; stages of a 64
// column slab of g (one box of 128 rows) and 64 rows of W (one box 64 wide);
// the accumulator is double-buffered in tensor memory so the epilogue of one
// tile overlaps the MMAs of the next.
constexpr int kQXK = 64, kQXStages = 4;
constexpr int kQXABytes = kTM * kQXK * 2;             // 16 KB
constexpr int kQXBBytes = kQXK * kTN * 2;             // 8 KB
constexpr int kQXStage = kQXABytes + kQXBBytes;
constexpr int kQXSmem = kQXStages * kQXStage + 1024;

template <typename T>
__global__ void __launch_bounds__(kQThreads, 2)
    linear_grad_x_tma_kernel(const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_w,
                             T* __restrict__ gx, long long M, int Cx, long long ntiles, int ntiles_n, int nk,
                             unsigned* __restrict__ status) {
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    __shared__ __align__(8) uint64_t full[kQXStages], empty[kQXStages], acc_full[2], acc_empty[2];
    __shared__ uint32_t taddr_s;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t ring = (smem_u32(tc_smem) + 1023u) & ~1023u;
    if (tid == 0) {
        for (int s = 0; s < kQXStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), 4);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kQMma) {  // two 64-column fp32 accumulators x 128 lanes
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&taddr_s)),
                     "r"(2 * kTN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = taddr_s;
    volatile int* abort = &s_abort;
    const long long my_tiles =
        static_cast<long long>(blockIdx.x) < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (warp == kQProducer) {
        if (lane == 0) {
            long long it = 0;
            for (long long lt = 0; lt < my_tiles && !*abort; ++lt) {
                const long long tile = blockIdx.x + lt * gridDim.x;
                const long long tm = tile / ntiles_n;
                const int n0 = static_cast<int>(tile - tm * ntiles_n) * kTN;
                const int m0 = static_cast<int>(tm * kTM);
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int s = static_cast<int>(it % kQXStages);
                    const uint32_t ph = static_cast<uint32_t>(it / kQXStages) & 1u;
                    if (!mbar_wait_or(smem_u32(&empty[s]), ph ^ 1u, abort)) break;
                    const uint32_t fb = smem_u32(&full[s]);
                    mbar_expect_tx(fb, kQXStage);
                    const uint32_t sa = ring + s * kQXStage, sb = sa + kQXABytes;
                    const int k0 = kc * kQXK;
                    tma_load_2d(sa, &map_g, k0, m0, fb);
                    tma_load_2d(sb, &map_w, n0, k0, fb);
                }
            }
        }
    } else if (warp == kQMma) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc<T>(kTM, kTN, 0, 1);
            long long it = 0;
            for (long long lt = 0; lt < my_tiles && !*abort; ++lt) {
                const int a = static_cast<int>(lt & 1);
                const uint32_t aph = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!mbar_wait_or(smem_u32(&acc_empty[a]), aph ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + a * kTN;
                bool ok = true;
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int s = static_cast<int>(it % kQXStages);
                    const uint32_t ph = static_cast<uint32_t>(it / kQXStages) & 1u;
                    if (!mbar_wait_or(smem_u32(&full[s]), ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = ring + s * kQXStage, sb = sa + kQXABytes;
#pragma unroll
                    for (int q = 0; q < kQXK / 16; ++q)  // A: 32 bytes along its rows; B: 16 rows of 128 bytes
                        umma_f16(d, umma_desc_sw128(sa + q * 32, 16, 1024), umma_desc_sw128(sb + q * 2048, kQXBBytes, 1024),
                                 idesc, kc > 0 || q > 0);
                    umma_commit(smem_u32(&empty[s]));  // the stage may be refilled once these MMAs are done
                }
                if (!ok) break;
                umma_commit(smem_u32(&acc_full[a]));
            }
        }
    } else {  // warps 0-3: read the accumulator back, round once, store
        for (long long lt = 0; lt < my_tiles; ++lt) {
            const int a = static_cast<int>(lt & 1);
            const uint32_t aph = static_cast<uint32_t>(lt >> 1) & 1u;
            if (!mbar_wait_or(smem_u32(&acc_full[a]), aph, abort)) break;
            tc_fence_after();
            const long long tile = blockIdx.x + lt * gridDim.x;
            const long long tm = tile / ntiles_n;
            const int n0 = static_cast<int>(tile - tm * ntiles_n) * kTN;
            const long long row = tm * kTM + warp * 32 + lane;
            const uint32_t lane_addr = tmem + a * kTN + (static_cast<uint32_t>(warp * 32) << 16);
            uint32_t r[2][32];
            tmem_ld32(lane_addr, r[0]);
            tmem_ld32(lane_addr + 32, r[1]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));  // the MMA warp may reuse this accumulator
            if (row < M) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int col = n0 + h * 32 + v * 8;
                        if (col >= Cx) continue;
                        uint4 o;
                        o.x = pack_pair<T>(__uint_as_float(r[h][8 * v + 0]), __uint_as_float(r[h][8 * v + 1]));
                        o.y = pack_pair<T>(__uint_as_float(r[h][8 * v + 2]), __uint_as_float(r[h][8 * v + 3]));
                        o.z = pack_pair<T>(__uint_as_float(r[h][8 * v + 4]), __uint_as_float(r[h][8 * v + 5]));
                        o.w = pack_pair<T>(__uint_as_float(r[h][8 * v + 6]), __uint_as_float(r[h][8 * v + 7]));
                        *reinterpret_cast<uint4*>(gx + row * Cx + col) = o;
                    }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort) atomicOr(status, kLinStatusTimeout);
    if (warp == kQMma) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTN));
}

// grad_W += g^T x and grad_b over one range of rows (split K): a CTA per
// 128 x 64 tile of grad_W and range; stages of 32 rows m: g^T (M-major) as two
// 64-wide boxes, x (N-major) as one, plus a constant second block of B (its
// first column all ones, the rest zero) so that D's column 64 sums g's columns
// (grad_b).  One accumulator of 80 columns.
constexpr int kQWK = 32, kQWStages = 6, kQWNB = 80;
constexpr int kQWABytes = kQWK * kUM * 2;             // 8 KB: two 64-wide blocks of 32 rows
constexpr int kQWBBytes = 2 * kQWK * 64 * 2;          // 8 KB: x's block and the constant block
constexpr int kQWStage = kQWABytes + kQWBBytes;
constexpr int kQWLoad = kQWABytes + kQWK * kUN * 2;   // bytes TMA writes per stage
constexpr int kQWSmem = kQWStages * kQWStage + 1024;

template <typename T>
__global__ void __launch_bounds__(kQThreads, 2)
    linear_grad_w_tma_kernel(const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_x,
                             float* __restrict__ wacc, float* __restrict__ bacc, unsigned* __restrict__ done,
                             unsigned* __restrict__ status, T* __restrict__ gw, T* __restrict__ gb, long long M, int P,
                             int Cx, int ntile, int ct, long long mchunk) {
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    __shared__ __align__(8) uint64_t full[kQWStages], empty[kQWStages], acc_full;
    __shared__ uint32_t taddr_s;
    __shared__ int s_abort;
    __shared__ unsigned ticket;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x % ntile;  // blocks of one split (the same rows) run together
    const long long split = blockIdx.x / ntile;
    const int tp = tile / ct, tc = tile - tp * ct;
    const int p0 = tp * kUM, c0 = tc * kUN;
    const long long mb = split * mchunk;
    const long long me = std::min<long long>(M, mb + mchunk);
    const int nk = static_cast<int>((me - mb + kQWK - 1) / kQWK);
    const uint32_t ring_off = ((smem_u32(tc_smem) + 1023u) & ~1023u) - smem_u32(tc_smem);
    const uint32_t ring = smem_u32(tc_smem) + ring_off;
    if (tid == 0) {
        for (int s = 0; s < kQWStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(&acc_full), 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kQMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&taddr_s)),
                     "r"(kUTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // B's constant block in every stage: row m holds a one in its first column, zeros elsewhere; under
    // the 128-byte swizzle the first 16-byte chunk of row m sits at chunk (m mod 8)
    for (int i = tid; i < kQWStages * kQWK * 8; i += kQThreads) {
        const int s = i / (kQWK * 8), r = i - s * (kQWK * 8), m = r >> 3, chunk = r & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (chunk == (m & 7)) v.x = pack_pair<T>(1.f, 0.f);
        *reinterpret_cast<uint4*>(tc_smem + ring_off + s * kQWStage + kQWABytes + kQWK * 128 + m * 128 + chunk * 16) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = taddr_s;
    volatile int* abort = &s_abort;

    if (warp == kQProducer) {
        if (lane == 0) {
            for (int j = 0; j < nk && !*abort; ++j) {
                const int s = j % kQWStages;
                const uint32_t ph = static_cast<uint32_t>(j / kQWStages) & 1u;
                if (!mbar_wait_or(smem_u32(&empty[s]), ph ^ 1u, abort)) break;
                const uint32_t fb = smem_u32(&full[s]);
                mbar_expect_tx(fb, kQWLoad);
                const uint32_t sa = ring + s * kQWStage, sb = sa + kQWABytes;
                // ranges are whole multiples of 32 rows, so a box never reaches into the next
                // range; past the last row of the matrix TMA fills zeros
                const int m = static_cast<int>(mb + static_cast<long long>(j) * kQWK);
                tma_load_2d(sa, &map_g, p0, m, fb);
                tma_load_2d(sa + kQWK * 128, &map_g, p0 + 64, m, fb);
                tma_load_2d(sb, &map_x, c0, m, fb);
            }
        }
    } else if (warp == kQMma) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc<T>(kUM, kQWNB, 1, 1);
            bool ok = true;
            for (int j = 0; j < nk; ++j) {
                const int s = j % kQWStages;
                const uint32_t ph = static_cast<uint32_t>(j / kQWStages) & 1u;
                if (!mbar_wait_or(smem_u32(&full[s]), ph, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = ring + s * kQWStage, sb = sa + kQWABytes;
#pragma unroll
                for (int q = 0; q < kQWK / 16; ++q)  // K = 16 rows of 128 bytes; the 64-wide blocks 4 KB apart
                    umma_f16(tmem, umma_desc_sw128(sa + q * 2048, kQWK * 128, 1024),
                             umma_desc_sw128(sb + q * 2048, kQWK * 128, 1024), idesc, j > 0 || q > 0);
                umma_commit(smem_u32(&empty[s]));
            }
            if (ok) umma_commit(smem_u32(&acc_full));
        }
    }
    // warps 0-3: the partial tile out (thread = row p), into the fp32 accumulators
    if (warp < 4) {
        const bool have = nk > 0 && mbar_wait_or(smem_u32(&acc_full), 0u, abort);
        tc_fence_after();
        const int p = p0 + warp * 32 + lane;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
        for (int h = 0; h < 3; ++h) {
            uint32_t r[32];
            tmem_ld32(lane_addr + h * 32, r);  // columns 64-95 hold grad_b in 64
            if (!have || p >= P) continue;
            if (h < 2) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const int col = c0 + h * 32 + v * 4;
                    if (col < Cx)
                        red_add4(wacc + static_cast<long long>(p) * Cx + col, __uint_as_float(r[4 * v]),
                                 __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                                 __uint_as_float(r[4 * v + 3]));
                }
            } else if (bacc != nullptr && tc == 0) {
                atomicAdd(bacc + p, __uint_as_float(r[0]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort) atomicOr(status, kLinStatusTimeout);
    if (warp == kQMma) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols));

    // The last CTA of this output tile rounds it once (its fence orders the other
    // CTAs' reductions, which precede their tickets, before its reads).
    __threadfence();
    __syncthreads();
    if (tid == 0) ticket = atomicAdd(done + tile, 1u);
    __syncthreads();
    if (ticket != gridDim.x / ntile - 1) return;
    __threadfence();
    round_tile<T, kQThreads>(wacc, bacc, gw, gb, P, Cx, p0, c0, tc == 0);
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms > 0 ? sms : 148;
}

// cuTensorMapEncodeTiled from the driver (resolved once through the runtime).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// A row-major [rows][cols] matrix of 16-bit elements as a 2-D tensor map with
// boxes 64 elements (128 bytes) wide and box_rows high, 128-byte swizzle, zeros
// outside the matrix.
bool swizzled_map(CUtensorMap* map, bool half, const void* base, long long rows, int cols, int box_rows) {
    const EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, half ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t linear_backward_typed(long long M, int P, int Cx, const void* x, const void* w, const void* gom,
                                  void* gx, void* gw, void* gb, float* ws, cudaStream_t stream) {
    constexpr bool kHalf = std::is_same<T, __half>::value;
    const int sms = device_sms();
    const long long wsz = static_cast<long long>(P) * Cx;
    float* wacc = ws;
    float* bacc = ws + wsz;
    unsigned* status = reinterpret_cast<unsigned*>(ws + wsz + P);
    unsigned* done = status + 1;  // one finishing counter per 128 x 64 tile of grad_W
    const long long ntile = static_cast<long long>((P + kUM - 1) / kUM) * ((Cx + kUN - 1) / kUN);
    // accumulators, the status word and the finishing counters
    cudaError_t e = cudaMemsetAsync(ws, 0, (wsz + P + 1 + ntile) * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (gx) {
        CUtensorMap map_g, map_w;
        if (!swizzled_map(&map_g, kHalf, gom, M, P, kTM) || !swizzled_map(&map_w, kHalf, w, P, Cx, kQXK))
            return cudaErrorInvalidValue;
        e = cudaFuncSetAttribute(linear_grad_x_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kQXSmem);
        if (e != cudaSuccess) return e;
        const int ntiles_n = (Cx + kTN - 1) / kTN;
        const long long ntiles = (M + kTM - 1) / kTM * ntiles_n;
        const int nk = (P + kQXK - 1) / kQXK;
        const long long grid = std::min<long long>(ntiles, 2LL * sms);
        linear_grad_x_tma_kernel<T><<<static_cast<unsigned>(grid), kQThreads, kQXSmem, stream>>>(
            map_g, map_w, static_cast<T*>(gx), M, Cx, ntiles, ntiles_n, nk, status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!gw && !gb) return cudaSuccess;
    CUtensorMap map_g, map_x;
    if (!swizzled_map(&map_g, kHalf, gom, M, P, kQWK) || !swizzled_map(&map_x, kHalf, x, M, Cx, kQWK))
        return cudaErrorInvalidValue;
    const int pt = (P + kUM - 1) / kUM, ct = (Cx + kUN - 1) / kUN;
    // split the rows (whole multiples of 32) so that the grid holds about two CTAs per SM
    const long long want = std::max<long long>(1, (2LL * sms + pt * ct - 1) / (pt * ct));
    long long mchunk = (M + want - 1) / want;
    mchunk = std::max<long long>(4LL * kQWK, (mchunk + kQWK - 1) / kQWK * kQWK);
    const long long splits = (M + mchunk - 1) / mchunk;
    const long long grid = splits * pt * ct;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(linear_grad_w_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kQWSmem);
    if (e != cudaSuccess) return e;
    linear_grad_w_tma_kernel<T><<<static_cast<unsigned>(grid), kQThreads, kQWSmem, stream>>>(
        map_g, map_x, wacc, gb ? bacc : nullptr, done, status, static_cast<T*>(gw), static_cast<T*>(gb), M, P, Cx,
        pt * ct, ct, mchunk);
    return cudaGetLastError();
}

}  // namespace

size_t linear_backward_workspace_bytes(int P, int Cx) {
    // grad_W and grad_b accumulators, the status word, one finishing counter per 128 x 64 tile
    const size_t ntile = static_cast<size_t>((P + kUM - 1) / kUM) * ((Cx + kUN - 1) / kUN);
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
