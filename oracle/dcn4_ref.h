/*
 * dcn4_ref.h — plain, slow CPU oracle for the DCNv4 core spatial aggregation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The product
 * path (libdcn4) never links, loads or calls it, and it shares no code, header,
 * table or helper with the GPU path.
 *
 * What it computes (CVPR'24 "Efficient Deformable ConvNets: Rethinking Dynamic
 * and Sparse Operator for Vision Applications", summarised on the CSDN page
 * "DCNv4论文解析", section 1.2 "回顾DCNv3" equation, with the softmax removed as in
 * section 2.1 "增强动态特性"):
 *
 *     y_g(p0) = sum_k  m_gk * x_g(p0 + p_k + offset_scale * dp_gk)
 *     y       = concat_g y_g                      (channels-last)
 *
 * x_g(.) is bilinear interpolation of group g's C' channels of the zero-extended
 * image (section 2.2, "GPU效率的理论分析": four coefficients per sampling point).
 * p_k enumerates a kh x kw convolution grid with stride / pad / dilation; with
 * remove_center the centre cell is skipped (DCNv4 module signature on the
 * mhpn.cn architecture page, "参数remove_center").
 *
 * Layouts (all dense, row-major, channels last):
 *   value        [N, H, W, G*Cg]
 *   offset_mask  [N, Ho, Wo, P]; group g owns entries [g*3K, (g+1)*3K):
 *                K pairs (dx_k, dy_k) followed by K masks m_k; [G*3K, P) is
 *                padding and is never read.
 *   out          [N, Ho, Wo, G*Cg]
 *   grad_*       same shape as the tensor they are the gradient of.
 *
 * Grid order: k runs over the kernel columns (x) in the outer loop and the
 * kernel rows (y) in the inner loop, i.e. k = iw*kh + ih before the centre is
 * removed; the centre cell (kw/2, kh/2) is skipped when remove_center != 0 and
 * later cells keep their relative order.  dx moves the sample along W, dy
 * along H.
 *
 * Sampling location for output (ho, wo), grid cell (ih, iw):
 *     h = ho*sh - ph + ih*dh + offset_scale*dy,   w = wo*sw - pw + iw*dw + offset_scale*dx
 * In location_fp32 mode the location is formed as one fp32 fused multiply-add
 * fmaf(offset_scale, d, base) — the precision in which the GPU kernels decide
 * which bilinear cell a sample falls in — and all later arithmetic stays in
 * double.  Otherwise the location is formed in double.
 *
 * Softmax variant (softmax != 0): the K masks of each (pixel, group) are
 * logits, normalised over k before they weigh the samples,
 *     m_gk -> exp(m_gk) / sum_j exp(m_gj)
 * — the DCNv3 aggregation the CSDN summary's section 1.2 equation gives, which
 * DCNv4 drops (section 2.1); the reference extension keeps it as a `softmax`
 * flag (mhpn.cn page, dcnv4_cuda_forward signature).  The exponentials are
 * taken after subtracting the largest logit (same value, no overflow).
 *
 * Element storage: REF_F32, REF_F16 (IEEE binary16), REF_BF16 (upper half of an
 * IEEE binary32) and REF_F64 (for finite-difference tests).  Every element is
 * decoded exactly into a double by this file's own bit-level decoders.
 * Outputs and gradients are written as double.
 */
#ifndef DCN4_REF_H
#define DCN4_REF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { REF_F32 = 0, REF_F16 = 1, REF_BF16 = 2, REF_F64 = 3 };

typedef struct {
    int N, H, W;          /* input batch and spatial size                      */
    int G, Cg;            /* groups and channels per group (C = G*Cg)          */
    int kh, kw;           /* kernel grid                                       */
    int sh, sw;           /* stride                                            */
    int ph, pw;           /* padding                                           */
    int dh, dw;           /* dilation                                          */
    double offset_scale;  /* multiplies the learned offsets only               */
    int remove_center;    /* 1: skip the centre grid cell (odd kh, kw only)    */
    int P;                /* row length of offset_mask, >= G*3K                */
    int dtype;            /* REF_* storage type of value/offset_mask/grad_out  */
    int location_fp32;    /* 1: form the sampling location with an fp32 fma    */
    int softmax;          /* 1: the masks are logits, normalised over k        */
} ref_problem;

/* Output size of the grid: Ho = (H + 2ph - (dh*(kh-1)+1)) / sh + 1 (floor).
 * Returns 0, or -1 when the problem is malformed. */
int ref_output_dims(const ref_problem* p, int* Ho, int* Wo);

/* Number of sampling points K = kh*kw - (remove_center ? 1 : 0). */
int ref_num_points(const ref_problem* p);

/* Forward: out[N,Ho,Wo,G*Cg] (double).  nthreads > 1 splits output rows
 * across std::thread workers; each output element is computed by one thread in the
 * same order.  Returns 0 or -1. */
int ref_forward(const ref_problem* p, const void* value, const void* offset_mask,
                double* out, int nthreads);

/* Backward for grad_out (stored in p->dtype):
 *   grad_value       [N,H,W,G*Cg]  = adjoint of the forward in value
 *   grad_offset_mask [N,Ho,Wo,P]   = d<grad_out, y>/d offset_mask; the padding
 *                                    tail [G*3K, P) is written as 0.
 * The bilinear derivative at an integer coordinate is the one-sided one of
 * the cell that floor() selects.  nthreads > 1 splits the batch across
 * std::thread workers (images are independent).  Returns 0 or -1. */
int ref_backward(const ref_problem* p, const void* value, const void* offset_mask,
                 const void* grad_out, double* grad_value, double* grad_offset_mask,
                 int nthreads);

/* Exact decode of n stored elements into doubles. */
void ref_decode(int dtype, const void* src, double* dst, int64_t n);

/* Store n doubles in `dtype`, each rounded to the nearest representable value,
 * ties to the one with an even last fraction bit (IEEE 754 roundTiesToEven);
 * beyond the largest finite value (by at least half a unit in its last place)
 * the result is an infinity; NaN stays NaN.  REF_F64 copies. */
void ref_encode(int dtype, const double* src, void* dst, int64_t n);

/* The merged offset/mask linear layer of the DCNv4 module (CSDN summary,
 * section 2.2 "DCN模块的微设计": the offsets and the dynamic weights come from a
 * single linear layer; with latency first, the depthwise convolution before it
 * is dropped):
 *     out[m, j] = round_dtype( sum_c x[m, c] * weight[j, c] + bias[j] )
 * for m < M rows (output pixels) and j < Cout (= P, the padded row length),
 * x [M, Cin] and weight [Cout, Cin] (nn.Linear layout) stored in `dtype`, bias
 * [Cout] in `dtype` or NULL (zero).  The sum is taken in double in c order and
 * rounded once (ref_encode).  Returns 0, or -1 for bad sizes. */
int ref_linear(int64_t M, int Cin, int Cout, int dtype, const void* x, const void* weight,
               const void* bias, void* out);

/* Gradients of ref_linear's affine map (before its rounding) for an upstream
 * gradient g [M, Cout] stored in `dtype`:
 *     grad_x[m, c] = sum_j g[m, j] * weight[j, c]      [M, Cin]
 *     grad_w[j, c] = sum_m g[m, j] * x[m, c]           [Cout, Cin]
 *     grad_b[j]    = sum_m g[m, j]                     [Cout]
 * in double, unrounded (the derivative of a linear map is its transpose; the
 * bias enters every row with weight 1).  Any of the three outputs may be NULL.
 * Rows of grad_x and rows of grad_w / grad_b are spread over nthreads threads.
 * Returns 0, or -1 for bad sizes. */
int ref_linear_backward(int64_t M, int Cin, int Cout, int dtype, const void* x, const void* weight, const void* g,
                        double* grad_x, double* grad_w, double* grad_b, int nthreads);

/* ---------------------------------------------------------------------------
 * Deformable attention, single scale (CSDN summary of "Efficient Deformable
 * ConvNets", section 1.1: each query attends to a selected number of key
 * sampling points whose positions and weights are set dynamically; section 1.2:
 * the weights are normalised with a softmax over the points, as in DCNv3).
 * For query q of image n and group g:
 *     y_g(q) = sum_{k<K} A_gk * x_g(r_q + offset_scale * dp_gk),
 *     A_gk   = exp(l_gk - max_j l_gj) / sum_j exp(l_gj - max_j l_gj)
 * with r_q the query's reference point (x, y) in pixel coordinates of value
 * (integer coordinates are pixel centres), dp_gk = (dx, dy) its K learned
 * offsets, l_gk its K attention logits, and x_g(.) the bilinear sample of the
 * zero-extended image (as the aggregation above).
 *   value          [N, H, W, G*Cg]     dtype
 *   ref_points     [N, Nq, 2]          fp32, (x, y)
 *   offset_logits  [N, Nq, P]          dtype: group g owns [g*3K, (g+1)*3K):
 *                                      K (dx, dy) pairs, then K logits
 *   out / grad_out [N, Nq, G*Cg]
 * --------------------------------------------------------------------------- */
typedef struct {
    int N, H, W;          /* value batch and spatial size                      */
    int G, Cg;            /* groups (heads) and channels per group             */
    int Nq, K;            /* queries per image, sampling points per query      */
    double offset_scale;  /* multiplies the learned offsets                     */
    int P;                /* row length of offset_logits, >= G*3K              */
    int dtype;            /* REF_* storage type of value/offset_logits/grad_out */
    int location_fp32;    /* 1: form the location with an fp32 fma             */
} ref_attn_problem;

/* Forward: out[N,Nq,G*Cg] (double).  nthreads > 1 splits queries across
 * std::thread workers.  Returns 0 or -1. */
int ref_attn_forward(const ref_attn_problem* p, const void* value, const float* ref_points,
                     const void* offset_logits, double* out, int nthreads);

/* Backward for grad_out: grad_value [N,H,W,G*Cg] (adjoint in value) and
 * grad_offset_logits [N,Nq,P]: d<grad_out, y>/d offsets and d/d logits
 * A_k (<gy, S_k> - sum_j A_j <gy, S_j>); the padding tail is 0.  The reference
 * points get no gradient.  nthreads > 1 splits the batch.  Returns 0 or -1. */
int ref_attn_backward(const ref_attn_problem* p, const void* value, const float* ref_points,
                      const void* offset_logits, const void* grad_out, double* grad_value,
                      double* grad_offset_logits, int nthreads);

#ifdef __cplusplus
}
#endif

#endif /* DCN4_REF_H */
