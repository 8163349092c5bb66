/*
 * dcn4.h — C ABI of libdcn4, the sm_100a (B200) DCNv4 core spatial aggregation.
 *
 * The operation (CSDN summary of "Efficient Deformable ConvNets: Rethinking
 * Dynamic and Sparse Operator for Vision Applications", section 1.2 equation,
 * with the softmax over K removed as section 2.1 "增强动态特性" describes):
 *
 *     y_g(p0) = sum_{k<K} m_gk * x_g(p0 + p_k + offset_scale * dp_gk),   y = concat_g y_g
 *
 * for every output pixel p0 and group g.  x_g(.) is bilinear interpolation of
 * the C' = Cg channels of group g (section 2.2: four coefficients per sample);
 * a bilinear corner outside the image contributes zero.  p_k runs over a
 * kh x kw convolution grid with stride, padding and dilation; remove_center
 * drops the centre cell so K = kh*kw - 1 (DCNv4 module / dcnv4_cuda_forward
 * signatures on the mhpn.cn architecture page).  The modulation scalars m_gk
 * are unbounded (no softmax) unless `softmax` is set, which gives the DCNv3
 * form: m_gk = exp(l_gk) / sum_j exp(l_gj) over the K mask entries l_gk of the
 * (pixel, group) (CSDN summary, section 1.2 DCNv3 equation; the `softmax` flag
 * of the dcnv4_cuda_forward signature on the mhpn.cn page).  The exponentials are taken
 * after subtracting the largest l_gj, in fp32 (expf), and grad_offset_mask
 * then holds the gradients of the logits l_gk:
 * m_gk * (<gy, S_k> - sum_j m_gj <gy, S_j>).
 *
 * Sampling location of grid cell (ih, iw) for output pixel (ho, wo):
 *     h = ho*sh - ph + ih*dh + offset_scale*dy,   w = wo*sw - pw + iw*dw + offset_scale*dx
 * formed in fp32 as fmaf(offset_scale, d, base) (one rounding).  The grid is
 * enumerated with the kernel column outer and the kernel row inner,
 * k = iw*kh + ih, skipping the centre (iw, ih) = (kw/2, kh/2) when
 * remove_center is set; dx moves along W and dy along H.
 *
 * Layouts (dense, contiguous, channels last; C = G*Cg):
 *   value            [N, H,  W,  C]   dtype
 *   offset_mask      [N, Ho, Wo, P]   dtype.  Group g owns entries [g*3K, (g+1)*3K):
 *                                     K pairs (dx_k, dy_k), then K masks m_k.
 *                                     Entries [G*3K, P) are padding: never read.
 *   out / grad_out   [N, Ho, Wo, C]   dtype
 *   grad_value       [N, H,  W,  C]   dtype
 *   grad_offset_mask [N, Ho, Wo, P]   dtype; the padding tail is written as 0.
 * P is a multiple of 8 and >= G*3K ("padded_offset_dim divisible by 8" on the
 * mhpn.cn page); dcn4_padded_offset_dim() gives the smallest such P.
 *
 * Precision: inputs are converted to fp32, every sum is accumulated in fp32,
 * and results are rounded once to dtype (round to nearest even).
 *
 * Ownership and execution: the caller owns every buffer (device memory) and
 * the stream.  The library allocates nothing and keeps no state between
 * calls; every call is asynchronous and ordered on `stream` (a cudaStream_t;
 * NULL is the legacy default stream).  Inputs must not alias outputs.
 *
 * Preconditions checked on the host before anything is launched (a failed
 * check launches nothing and returns a negative status):
 *   - non-NULL pointers (except when N == 0, which is a successful no-op);
 *   - every pointer 16-byte aligned;
 *   - Cg * sizeof(dtype) a multiple of 16 bytes (fp32: Cg % 4 == 0, fp16/bf16:
 *     Cg % 8 == 0) and Cg * sizeof(dtype) / 32 (rounded up) a power of two <= 32;
 *   - H, W < 2^24 and H*W*C < 2^31 (per image), Ho >= 1, Wo >= 1;
 *   - remove_center only with odd kh and kw;
 *   - remove_center and softmax each 0 or 1.
 * Errors are returned, never raised: no abort, no exception, no device trap.
 */
#ifndef DCN4_H
#define DCN4_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DCN4_VERSION 160  /* 1.6.0: the output projection fused behind the sampler (dcn4_forward_proj) */

typedef enum {
    DCN4_F32 = 0,   /* IEEE binary32            */
    DCN4_F16 = 1,   /* IEEE binary16            */
    DCN4_BF16 = 2   /* bfloat16 (upper half of binary32) */
} dcn4_dtype;

typedef enum {
    DCN4_OK = 0,
    DCN4_ERR_NULL = -1,         /* a required pointer is NULL                         */
    DCN4_ERR_BAD_SHAPE = -2,    /* non-positive size, empty output grid, bad geometry */
    DCN4_ERR_BAD_P = -3,        /* P < G*3K or P not a multiple of 8                  */
    DCN4_ERR_MISALIGNED = -4,   /* a pointer is not 16-byte aligned                   */
    DCN4_ERR_UNSUPPORTED = -5,  /* valid operator, but outside this build's kernels   */
    DCN4_ERR_WORKSPACE = -6,    /* workspace missing or smaller than required         */
    DCN4_ERR_LAUNCH = -7,       /* the CUDA launch failed; see dcn4_last_error()      */
    DCN4_ERR_DTYPE = -8         /* dtype is not a dcn4_dtype                          */
} dcn4_status;

/* Geometry of one call.  All fields are read, none is written. */
typedef struct {
    int N, H, W;          /* value is [N, H, W, G*Cg]                           */
    int G, Cg;            /* groups, channels per group                         */
    int kh, kw;           /* sampling grid (kernel) size                        */
    int sh, sw;           /* stride  (>= 1)                                     */
    int ph, pw;           /* padding (>= 0)                                     */
    int dh, dw;           /* dilation (>= 1)                                    */
    float offset_scale;   /* multiplies the learned offsets, not the grid      */
    int remove_center;    /* 0 or 1                                             */
    int P;                /* row length of offset_mask / grad_offset_mask       */
    int dtype;            /* dcn4_dtype of every tensor argument                */
    int softmax;          /* 0: masks used as given; 1: softmax over the K masks
                             of each (pixel, group) (DCNv3 form)                */
} dcn4_params;

/* Library version (DCN4_VERSION of the build). */
int dcn4_version(void);

/* Number of sampling points K = kh*kw - remove_center, or a negative status. */
int dcn4_num_points(const dcn4_params* p);

/* Smallest valid P for G groups of K points: G*3K rounded up to a multiple of 8.
 * Returns a negative status for G < 1 or K < 1. */
int dcn4_padded_offset_dim(int G, int K);

/* Output grid: Ho = (H + 2*ph - (dh*(kh-1) + 1)) / sh + 1 (floor), likewise Wo.
 * Writes *Ho, *Wo and returns DCN4_OK, or a negative status. */
int dcn4_output_dims(const dcn4_params* p, int* Ho, int* Wo);

/* Host-only validation of p (shape, P, dtype, supported sizes); touches no
 * GPU.  Returns DCN4_OK or the status dcn4_forward would return. */
int dcn4_check_params(const dcn4_params* p);

/* Forward: out = y.  Reads value and offset_mask, writes every element of out.
 * One kernel launch on `stream`. */
int dcn4_forward(const dcn4_params* p, const void* value, const void* offset_mask, void* out,
                 void* stream);

/* Forward with its producer fused in: the merged offset/mask linear layer of
 * the DCNv4 module (CSDN summary, section 2.2 "DCN模块的微设计": one linear layer
 * gives the offsets and the dynamic weights; with latency first the depthwise
 * convolution before it is dropped), then the aggregation:
 *     offset_mask[n, ho, wo, j] = round_dtype( sum_c x[n, ho, wo, c] * weight[j, c] + bias[j] )
 *     out = dcn4_forward(value, offset_mask)
 * formed tile by tile in the kernel (tensor cores, fp32 accumulation, the bias
 * added in fp32, one rounding to dtype), so the offset_mask is never read from
 * HBM.  One kernel launch on `stream`.
 *   x                [N, Ho, Wo, Cx]  dtype: the features of each output pixel
 *   weight           [P, Cx]          dtype (nn.Linear layout: row j gives entry j)
 *   bias             [P]              dtype, or NULL for none
 *   out              [N, Ho, Wo, C]   dtype
 *   offset_mask_out  [N, Ho, Wo, P]   dtype, or NULL: receives the offset_mask the
 *                                     samples used (for a later dcn4_backward)
 * Rows [G*3K, P) of weight give the padding entries: computed (and stored in
 * offset_mask_out), never sampled.  fp16 and bf16 only (DCN4_ERR_UNSUPPORTED for
 * fp32); Cx a multiple of 16 (DCN4_ERR_BAD_SHAPE otherwise) whose staged tiles
 * fit shared memory (DCN4_ERR_UNSUPPORTED otherwise); every non-NULL pointer
 * 16-byte aligned.  The same checks as dcn4_forward otherwise. */
int dcn4_forward_linear(const dcn4_params* p, int Cx, const void* value, const void* x, const void* weight,
                        const void* bias, void* out, void* offset_mask_out, void* stream);

/* Bytes of device workspace dcn4_backward needs, each part rounded up to 256
 * bytes: a header of 32-bit words (4 fallback counters, one word per image,
 * and for fp16/bf16 one record counter per grad_value tile), one 32-bit cell
 * box per output pixel (N*Ho*Wo), then
 *   fp32:      a 2-byte cell code per sample (N*Ho*Wo*G*K of them);
 *   fp16/bf16: per grad_value tile, room for bcap 12-byte sample records
 *              (4-byte output pixel + 8 bytes of bin, mask bits and
 *              fixed-point bilinear fractions), where the tiles and bcap
 *              follow from the shape (about 1.06x the records a tile
 *              expects, + 512);
 * 0 if p is invalid. */
size_t dcn4_backward_workspace_size(const dcn4_params* p);

/* Backward of the forward for upstream gradient grad_out:
 *   grad_value       = sum over samples of m_gk * bilinear_weight * grad_out (scatter-add)
 *   grad_offset_mask = (d/d dx, d/d dy) = offset_scale * m_gk * <grad_out, dS/dw, dS/dh>
 *                      and d/d m_gk = <grad_out, S> per (pixel, group, k);
 * S is the bilinear sample, and its derivative at an integer coordinate is the
 * one of the cell floor() selects.  Both gradients are overwritten (not
 * accumulated into); the offset_mask padding tail is written as 0.
 * `workspace` (device, 16-byte aligned, >= dcn4_backward_workspace_size bytes)
 * is scratch, clobbered by the call: it receives, per image, how far any
 * sample reaches from its grid position, and per sample its bilinear cell
 * (fp32: relative to its grid position; fp16/bf16: filed, with its weights,
 * under every grad_value tile whose cells hold it).
 * Launches, on `stream`: a memset of the per-image words (and, for fp16/bf16,
 * one of the per-tile counters), one kernel for grad_offset_mask (and the
 * workspace), and one for grad_value.  grad_value is not scattered with
 * atomics: each element is summed by one thread in fp32 (over the samples
 * sorted by cell) and written once, so results are deterministic up to the
 * order in which samples of one cell are added. */
int dcn4_backward(const dcn4_params* p, const void* value, const void* offset_mask,
                  const void* grad_out, void* grad_value, void* grad_offset_mask,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Backward without a caller-provided workspace.
 *
 * This entry point has no counterpart in the paper: it exists for callers that
 * cannot give the library device memory when they call it, such as a plugin
 * inside a host runtime that owns every device buffer and offers no
 * allocator, or a service that fixes its device-memory budget at start-up.
 * It computes exactly what dcn4_backward computes, taking its scratch from a
 * fixed area that this library reserves on every device that loads it
 * (DCN4_NOALLOC_SCRATCH_BYTES, 64 MiB, held until the process exits); it calls
 * no cudaMalloc, cudaFree or allocating library routine.
 *   - Sizes: the problem's dcn4_backward_workspace_size must not exceed
 *     dcn4_backward_noalloc_capacity(); larger problems are rejected with
 *     DCN4_ERR_WORKSPACE before anything is launched (detail in
 *     dcn4_noalloc_last_error()).
 *   - Set-up: the first call on a device (made with that device current) looks
 *     up the area's device address, and so does the first call after a device
 *     reset (a new context); make such a call before any stream capture begins.
 *   - Sharing: every call on a device uses the same area, which keeps the
 *     last call's contents (each call resets what it needs).  Calls whose
 *     executions overlap on the GPU (different streams, no ordering between
 *     them) race on the area and give wrong results: order them.
 * Arguments, layouts, errors and launches are those of dcn4_backward. */
#define DCN4_NOALLOC_SCRATCH_BYTES (64u << 20)

int dcn4_backward_noalloc(const dcn4_params* p, const void* value, const void* offset_mask,
                          const void* grad_out, void* grad_value, void* grad_offset_mask, void* stream);

/* Bytes of scratch dcn4_backward_noalloc can use (DCN4_NOALLOC_SCRATCH_BYTES). */
size_t dcn4_backward_noalloc_capacity(void);

/* Detail of the last failing dcn4_backward_noalloc size or set-up check on
 * this host thread ("" if none; launch errors are in dcn4_last_error()). */
const char* dcn4_noalloc_last_error(void);

/* The two stages of dcn4_backward, callable on their own (same arguments,
 * layouts and errors as dcn4_backward):
 *   dcn4_backward_offset_mask writes grad_offset_mask and fills `workspace`
 *     (the per-image reach, per-pixel cell boxes, and the per-sample cell
 *     codes or per-tile records); launches the memsets and one kernel.
 *   dcn4_backward_value writes grad_value from offset_mask, grad_out and a
 *     workspace filled by dcn4_backward_offset_mask for the same offset_mask
 *     (and the same params), ordered before it; one kernel.
 * dcn4_backward(...) is dcn4_backward_offset_mask(...) then
 * dcn4_backward_value(...) on the same stream. */
int dcn4_backward_offset_mask(const dcn4_params* p, const void* value, const void* offset_mask,
                              const void* grad_out, void* grad_offset_mask, void* workspace,
                              size_t workspace_bytes, void* stream);
int dcn4_backward_value(const dcn4_params* p, const void* offset_mask, const void* grad_out,
                        void* grad_value, const void* workspace, size_t workspace_bytes, void* stream);

/* Fallback counters of the last dcn4_backward (or dcn4_backward_value) run on
 * `workspace` for the same params: counts[0] = grad_value tiles whose filed
 * sample records failed the kernel's consistency checks (each such tile is
 * recomputed by the direct path, so the gradient stays exact; a nonzero count
 * means a filing fault), counts[1] = tiles that rescanned the offsets instead
 * of reading their records (bucket overflow, samples beyond the filing
 * window, or images of very large reach), counts[2] = tiles that took the
 * direct path for any reason.  Copies 16 bytes from the workspace to the host
 * on `stream` and waits for it (the one synchronising call of the library).
 * Same checks as dcn4_backward; counts must hold 3 ints. */
int dcn4_backward_diagnostics(const dcn4_params* p, const void* workspace, size_t workspace_bytes, int* counts,
                              void* stream);

/* Bytes of device workspace dcn4_backward_linear needs: dcn4_backward's
 * workspace rounded up to 256 bytes, then fp32 accumulators for grad_weight
 * (P*Cx) and grad_bias (P), a 32-bit status word (nonzero after the call if a
 * bounded wait inside the linear kernels gave up; the outputs are then not
 * valid) and one 32-bit counter per 128 x 64 tile of grad_weight, rounded up
 * to 256 bytes; 0 if p is invalid. */
size_t dcn4_backward_linear_workspace_size(const dcn4_params* p, int Cx);

/* Backward of dcn4_forward_linear, the aggregation with its offset/mask linear
 * layer (CSDN summary, section 2.2 "DCN模块的微设计"): with
 * offset_mask = x weight^T + bias as saved by the forward (its offset_mask_out),
 *   grad_value, grad_offset_mask  as dcn4_backward computes them, then, with
 *   g = grad_offset_mask as an [M = N*Ho*Wo, P] matrix (its padding columns are 0):
 *   grad_x      [N, Ho, Wo, Cx] = g weight          (sum over j of g[m, j] * weight[j, c])
 *   grad_weight [P, Cx]         = g^T x             (sum over m of g[m, j] * x[m, c])
 *   grad_bias   [P]             = sum over m of g[m, j]
 * All of dtype (fp16 or bf16; DCN4_ERR_UNSUPPORTED for fp32).  The products read
 * g as dcn4_backward rounded it to dtype, run on the tensor cores (tcgen05, fed
 * by TMA) with fp32 accumulation and are rounded to dtype once; grad_weight and
 * grad_bias sum partial products of row chunks with fp32 atomics (so their last
 * bit may vary from call to call).  grad_x, grad_weight and grad_bias may each be NULL (not
 * wanted); grad_value and grad_offset_mask are required.  Every pointer 16-byte
 * aligned; Cx a positive multiple of 16 (DCN4_ERR_BAD_SHAPE); `workspace`
 * (device, >= dcn4_backward_linear_workspace_size bytes) is clobbered, its first
 * part exactly as by dcn4_backward (so dcn4_backward_diagnostics reads it).
 * N*Ho*Wo and P*Cx must be below 2^31 (DCN4_ERR_UNSUPPORTED).  With N*Ho*Wo = 0
 * only grad_weight and grad_bias are written (zeros).
 * Launches on `stream`: dcn4_backward's launches, then a memset of the linear
 * part of the workspace, one kernel for grad_x and one for grad_weight and
 * grad_bias (which also rounds them). */
int dcn4_backward_linear(const dcn4_params* p, int Cx, const void* value, const void* offset_mask, const void* x,
                         const void* weight, const void* grad_out, void* grad_value, void* grad_offset_mask,
                         void* grad_x, void* grad_weight, void* grad_bias, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Forward with the output projection fused behind it: the DCNv4 module puts a
 * linear layer on each side of the core operator (CSDN summary, section 2.2
 * "DCN模块的微设计", which merges the layers around the core); this is the
 * aggregation followed by the one after it:
 *     core = dcn4_forward(value, offset_mask)          (rounded to dtype)
 *     out[n, ho, wo, o] = round_dtype( sum_c core[n, ho, wo, c] * weight[o, c] + bias[o] )
 * formed tile by tile in the kernel: the sampling threads leave the tile's core
 * rows in shared memory, the tensor cores (tcgen05, fp32 accumulation in tensor
 * memory) multiply them by weight, the bias is added in fp32 and the result
 * rounded once, so the core output need not go through HBM.  One kernel launch
 * on `stream`.
 *   offset_mask [N, Ho, Wo, P]     dtype, as for dcn4_forward
 *   weight      [Cout, C]          dtype (nn.Linear layout: row o gives output o)
 *   bias        [Cout]             dtype, or NULL for none
 *   out         [N, Ho, Wo, Cout]  dtype
 *   core_out    [N, Ho, Wo, C]     dtype, or NULL: receives the core output (for
 *                                  a later dcn4_backward_proj)
 * fp16 and bf16 only (DCN4_ERR_UNSUPPORTED for fp32).  Cout a positive multiple
 * of 16 (DCN4_ERR_BAD_SHAPE), at most 128 (DCN4_ERR_UNSUPPORTED: the kernel
 * forms M = 128 rows of weight per tile against the tile's pixels).  It needs
 * C a multiple of 64 up to 256 and tiles of 16, 32 or 64 pixels (the power of
 * two of pixels that 256 threads over the groups' channel slices give, fewer
 * for long offset_mask rows: C = 64 with G = 4, C = 128 with G = 4 or 8 and
 * C = 256 with G = 16 give 64, 32 and 16); DCN4_ERR_UNSUPPORTED otherwise, or
 * when the tiles do not fit shared memory.  Every non-NULL pointer 16-byte aligned.  The
 * same checks as dcn4_forward otherwise.  A bounded wait of the tensor-core
 * step that gives up sets the status word dcn4_forward_tc_status reads. */
int dcn4_forward_proj(const dcn4_params* p, int Cout, const void* value, const void* offset_mask, const void* weight,
                      const void* bias, void* out, void* core_out, void* stream);

/* The status word of the forward's tensor-core steps (dcn4_forward_linear's
 * tcgen05 producer and dcn4_forward_proj): 0 while every wait on the tensor
 * cores has completed, nonzero once one gave up (its tile's results are then
 * not written).  Synchronous (waits for the device); reset != 0 clears it.
 * Returns the word, or a negative DCN4_ERR_* status if it cannot be read. */
int dcn4_forward_tc_status(int reset);

/* Bytes of device workspace dcn4_backward_proj needs: dcn4_backward's, then
 * room for the gradient of the core output (N*Ho*Wo*C elements of dtype), then
 * the projection's fp32 accumulators and counters, each rounded up to 256
 * bytes; 0 if p is invalid. */
size_t dcn4_backward_proj_workspace_size(const dcn4_params* p, int Cout);

/* Backward of dcn4_forward_proj.  With core = the core output the forward saved
 * (its core_out) and g = grad_out [M = N*Ho*Wo, Cout]:
 *   grad_core   [N, Ho, Wo, C]  = g weight      (in the workspace, rounded to dtype)
 *   grad_weight [Cout, C]       = g^T core
 *   grad_bias   [Cout]          = sum over m of g[m, o]
 *   grad_value, grad_offset_mask = dcn4_backward(value, offset_mask, grad_core)
 * All of dtype (fp16 or bf16; DCN4_ERR_UNSUPPORTED for fp32).  The products run
 * on the tensor cores (tcgen05, fed by TMA) with fp32 accumulation, rounded to
 * dtype once; grad_weight and grad_bias sum row chunks with fp32 atomics (their
 * last bit may vary from call to call).  grad_weight and grad_bias may be NULL
 * (not wanted; core_out is needed only for grad_weight); grad_value and
 * grad_offset_mask are required.  Every pointer 16-byte aligned; Cout and C
 * multiples of 16 (DCN4_ERR_BAD_SHAPE); N*Ho*Wo and Cout*C below 2^31
 * (DCN4_ERR_UNSUPPORTED); `workspace` (device, >= dcn4_backward_proj_workspace_size
 * bytes) is clobbered, its first part exactly as by dcn4_backward (so
 * dcn4_backward_diagnostics reads it).  With N*Ho*Wo = 0 only grad_weight and
 * grad_bias are written (zeros).  Launches on `stream`: a memset and one or two
 * kernels for the projection's gradients, then dcn4_backward's launches. */
int dcn4_backward_proj(const dcn4_params* p, int Cout, const void* value, const void* offset_mask,
                       const void* core_out, const void* weight, const void* grad_out, void* grad_value,
                       void* grad_offset_mask, void* grad_weight, void* grad_bias, void* workspace,
                       size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Deformable attention, single scale.
 *
 * The pages describe deformable attention as letting each query attend to a
 * selected number of key sampling points whose positions and weights are
 * determined dynamically (CSDN summary of "Efficient Deformable ConvNets",
 * section 1.1), and note that the aggregation's memory optimisations apply to
 * it (section 2.2, "消除冗余内存指令").  This is that operation on one feature
 * map, with the weights normalised by a softmax over the points as in the
 * DCNv3 equation of section 1.2:
 *
 *     y_g(q) = sum_{k<K} A_gk * x_g(r_q + offset_scale * dp_gk),
 *     A_gk   = exp(l_gk - max_j l_gj) / sum_j exp(l_gj - max_j l_gj)
 *
 * for every query q (reference point r_q) and group g (a head).  x_g(.) is the
 * bilinear sample of the zero-extended map exactly as in dcn4_forward, the
 * location formed in fp32 as fmaf(offset_scale, d, r), the exponentials in fp32
 * (expf), sums in fp32, one rounding of each result to dtype.
 *
 * Layouts (dense, contiguous; C = G*Cg):
 *   value              [N, H, W, C]    dtype
 *   ref_points         [N, Nq, 2]      fp32 (x, y) in pixel coordinates of value;
 *                                      integer coordinates are pixel centres
 *   offset_logits      [N, Nq, P]      dtype.  Group g owns [g*3K, (g+1)*3K):
 *                                      K pairs (dx, dy), then K logits l_k.
 *                                      Entries [G*3K, P) are padding: never read.
 *   out / grad_out     [N, Nq, C]      dtype
 *   grad_value         [N, H, W, C]    dtype
 *   grad_offset_logits [N, Nq, P]      dtype; the padding tail is written as 0.
 * The reference points receive no gradient.  Preconditions as for dcn4_forward
 * (16-byte aligned pointers, Cg*sizeof(dtype) a multiple of 16 and /32 a power
 * of two, P >= G*3K a multiple of 8), plus K <= 1024 points whose rows fit
 * shared memory; N*Nq == 0 is a successful no-op.
 * ------------------------------------------------------------------------- */
typedef struct {
    int N, H, W;          /* value is [N, H, W, G*Cg]                          */
    int G, Cg;            /* groups (heads), channels per group                */
    int Nq, K;            /* queries per image, sampling points per query      */
    float offset_scale;   /* multiplies the offsets                             */
    int P;                /* row length of offset_logits / grad_offset_logits  */
    int dtype;            /* dcn4_dtype of every tensor argument but ref_points */
} dcn4_attn_params;

/* Host-only validation of p; returns DCN4_OK or the status a call would return. */
int dcn4_attn_check_params(const dcn4_attn_params* p);

/* Forward: out = y.  One kernel launch on `stream`. */
int dcn4_attn_forward(const dcn4_attn_params* p, const void* value, const float* ref_points,
                      const void* offset_logits, void* out, void* stream);

/* Bytes of workspace dcn4_attn_backward needs: 0 for fp32, else an fp32
 * accumulator for grad_value (N*H*W*C*4, rounded up to 256); 0 if p is invalid. */
size_t dcn4_attn_backward_workspace_size(const dcn4_attn_params* p);

/* Backward for grad_out: grad_value (overwritten) and grad_offset_logits
 * (overwritten): d/d dx_k = offset_scale * A_k * <gy, dS/dw>, likewise dy, and
 * d/d l_k = A_k (<gy, S_k> - sum_j A_j <gy, S_j>).  grad_value is scattered
 * with fp32 vector reductions (red.global.add.v4.f32) into the workspace (into
 * grad_value itself for fp32), so the order of its sums, and its last bits,
 * may differ between calls.  Launches, on `stream`: a memset of the
 * accumulator, one kernel, and for fp16/bf16 one rounding kernel. */
int dcn4_attn_backward(const dcn4_attn_params* p, const void* value, const float* ref_points,
                       const void* offset_logits, const void* grad_out, void* grad_value,
                       void* grad_offset_logits, void* workspace, size_t workspace_bytes, void* stream);

/* Name of a dcn4_status. */
const char* dcn4_status_string(int status);

/* Detail of the last failing call on this host thread ("" if none). */
const char* dcn4_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DCN4_H */
