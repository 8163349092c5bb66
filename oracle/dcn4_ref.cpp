// dcn4_ref.cpp — plain CPU oracle of the DCNv4 core spatial aggregation.
//
// TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).  See
// dcn4_ref.h for the operation, layouts and the readings it takes.  Every step
// is written out in the order the definition states it: no blocking, fusion or
// reordering.  Accumulation is in double.
#include "dcn4_ref.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include <thread>

namespace {

// ---------------------------------------------------------------------------
// Exact element decoders (own bit-level definitions, IEEE 754-2008 formats).
// ---------------------------------------------------------------------------

// binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double decode_f16(uint16_t bits) {
    const int sign = bits >> 15;
    const int expo = (bits >> 10) & 0x1f;
    const int frac = bits & 0x3ff;
    double mag;
    if (expo == 0) {
        mag = std::ldexp(static_cast<double>(frac), -24);            // subnormal: frac * 2^-24
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = std::ldexp(static_cast<double>(frac | 0x400), expo - 25);  // 1.frac * 2^(e-15)
    }
    return sign ? -mag : mag;
}

// bfloat16: the upper 16 bits of a binary32.
double decode_bf16(uint16_t bits) {
    const uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// Encoders: the nearest representable value, ties to an even last fraction bit.
// std::nearbyint rounds to an integer in the default mode (to nearest, ties to
// even); a / 2^k is exact, so q below is the value in units of the last place.

// binary16: normal numbers 1.f x 2^E (E in [-14, 15], 10 fraction bits, unit in
// the last place 2^(E-10)); below 2^-14 the unit is 2^-24 (subnormals).
uint16_t encode_f16(double v) {
    if (std::isnan(v)) return 0x7e00;
    const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
    const double a = std::fabs(v);
    if (a == 0.0) return sign;
    if (std::isinf(a)) return sign | 0x7c00;
    int e;
    std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1): the leading bit is 2^(e-1)
    int E = e - 1;
    if (E < -14) {
        const double q = std::nearbyint(std::ldexp(a, 24));  // units of 2^-24, <= 1024
        return sign | static_cast<uint16_t>(q);              // q = 1024 is the smallest normal
    }
    double q = std::nearbyint(std::ldexp(a, 10 - E));        // in [1024, 2048]
    if (q == 2048.0) {
        q = 1024.0;
        ++E;
    }
    if (E > 15) return sign | 0x7c00;
    return sign | static_cast<uint16_t>(((E + 15) << 10) | (static_cast<int>(q) - 1024));
}

// bfloat16: binary32's exponent range (E in [-126, 127]) with 7 fraction bits;
// below 2^-126 the unit is 2^-133.
uint16_t encode_bf16(double v) {
    if (std::isnan(v)) return 0x7fc0;
    const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
    const double a = std::fabs(v);
    if (a == 0.0) return sign;
    if (std::isinf(a)) return sign | 0x7f80;
    int e;
    std::frexp(a, &e);
    int E = e - 1;
    if (E < -126) {
        const double q = std::nearbyint(std::ldexp(a, 133));  // <= 128
        return sign | static_cast<uint16_t>(q);
    }
    double q = std::nearbyint(std::ldexp(a, 7 - E));          // in [128, 256]
    if (q == 256.0) {
        q = 128.0;
        ++E;
    }
    if (E > 127) return sign | 0x7f80;
    return sign | static_cast<uint16_t>(((E + 127) << 7) | (static_cast<int>(q) - 128));
}

void store(void* buf, int dtype, int64_t i, double v) {
    switch (dtype) {
        case REF_F32: static_cast<float*>(buf)[i] = static_cast<float>(v); break;  // C rounds to nearest even
        case REF_F16: static_cast<uint16_t*>(buf)[i] = encode_f16(v); break;
        case REF_BF16: static_cast<uint16_t*>(buf)[i] = encode_bf16(v); break;
        case REF_F64: static_cast<double*>(buf)[i] = v; break;
        default: break;
    }
}

double load(const void* buf, int dtype, int64_t i) {
    switch (dtype) {
        case REF_F32: return static_cast<double>(static_cast<const float*>(buf)[i]);
        case REF_F16: return decode_f16(static_cast<const uint16_t*>(buf)[i]);
        case REF_BF16: return decode_bf16(static_cast<const uint16_t*>(buf)[i]);
        case REF_F64: return static_cast<const double*>(buf)[i];
        default: return NAN;
    }
}

bool valid(const ref_problem* p) {
    if (!p) return false;
    if (p->N < 0 || p->H <= 0 || p->W <= 0 || p->G <= 0 || p->Cg <= 0) return false;
    if (p->kh <= 0 || p->kw <= 0 || p->sh <= 0 || p->sw <= 0 || p->dh <= 0 || p->dw <= 0) return false;
    if (p->ph < 0 || p->pw < 0) return false;
    if (p->remove_center && ((p->kh % 2) == 0 || (p->kw % 2) == 0)) return false;
    if (p->dtype < REF_F32 || p->dtype > REF_F64) return false;
    const int K = p->kh * p->kw - (p->remove_center ? 1 : 0);
    if (K <= 0 || p->P < p->G * 3 * K) return false;
    return true;
}

int out_dims(const ref_problem* p, int* Ho, int* Wo) {
    const int eff_h = p->dh * (p->kh - 1) + 1;
    const int eff_w = p->dw * (p->kw - 1) + 1;
    const int num_h = p->H + 2 * p->ph - eff_h;
    const int num_w = p->W + 2 * p->pw - eff_w;
    if (num_h < 0 || num_w < 0) return -1;
    *Ho = num_h / p->sh + 1;
    *Wo = num_w / p->sw + 1;
    return 0;
}

// One grid cell of the sampling grid p_k, in k order.
struct Cell {
    int ih, iw;
};

// k order: kernel columns outer, kernel rows inner; the centre cell is dropped
// when remove_center is set, the rest keep their order.
std::vector<Cell> grid_cells(const ref_problem* p) {
    std::vector<Cell> cells;
    for (int iw = 0; iw < p->kw; ++iw) {
        for (int ih = 0; ih < p->kh; ++ih) {
            if (p->remove_center && ih == p->kh / 2 && iw == p->kw / 2) continue;
            cells.push_back(Cell{ih, iw});
        }
    }
    return cells;
}

// p0 + p_k + s*dp: the sampling location of one point.
void sample_location(const ref_problem* p, int ho, int wo, const Cell& c, double dx,
                     double dy, double* h, double* w) {
    const int base_h = ho * p->sh - p->ph + c.ih * p->dh;
    const int base_w = wo * p->sw - p->pw + c.iw * p->dw;
    if (p->location_fp32) {
        const float s = static_cast<float>(p->offset_scale);
        *h = static_cast<double>(std::fmaf(s, static_cast<float>(dy), static_cast<float>(base_h)));
        *w = static_cast<double>(std::fmaf(s, static_cast<float>(dx), static_cast<float>(base_w)));
    } else {
        *h = static_cast<double>(base_h) + p->offset_scale * dy;
        *w = static_cast<double>(base_w) + p->offset_scale * dx;
    }
}

// Bilinear cell of a location: the four corners (h0 + a, w0 + b), a, b in {0, 1},
// with weights (a ? lh : 1-lh) * (b ? lw : 1-lw).  A location with h < -1,
// h >= H, w < -1 or w >= W touches no pixel of the image (every corner is
// outside), so it is reported as "no cell".
struct Bilinear {
    bool any;
    int h0, w0;
    double lh, lw;
};

Bilinear bilinear_cell(const ref_problem* p, double h, double w) {
    Bilinear b{};
    b.any = (h >= -1.0 && h < static_cast<double>(p->H) && w >= -1.0 &&
             w < static_cast<double>(p->W));
    if (!b.any) return b;
    const double fh = std::floor(h);
    const double fw = std::floor(w);
    b.h0 = static_cast<int>(fh);
    b.w0 = static_cast<int>(fw);
    b.lh = h - fh;
    b.lw = w - fw;
    return b;
}

bool inside(const ref_problem* p, int y, int x) {
    return y >= 0 && y < p->H && x >= 0 && x < p->W;
}

// Index of value[n, y, x, g*Cg + c].
int64_t value_index(const ref_problem* p, int n, int y, int x, int g, int c) {
    const int64_t C = static_cast<int64_t>(p->G) * p->Cg;
    return ((static_cast<int64_t>(n) * p->H + y) * p->W + x) * C + static_cast<int64_t>(g) * p->Cg + c;
}

// x_g at a fractional location for channel c of group g (zero-extended image).
double sample_value(const ref_problem* p, const void* value, int n, int g, int c,
                    const Bilinear& b) {
    if (!b.any) return 0.0;
    double s = 0.0;
    for (int a = 0; a < 2; ++a) {
        for (int bb = 0; bb < 2; ++bb) {
            const int y = b.h0 + a;
            const int x = b.w0 + bb;
            if (!inside(p, y, x)) continue;
            const double wt = (a ? b.lh : 1.0 - b.lh) * (bb ? b.lw : 1.0 - b.lw);
            s += wt * load(value, p->dtype, value_index(p, n, y, x, g, c));
        }
    }
    return s;
}

// Runs body(i) for i in [0, count), splitting the range into contiguous
// chunks over nthreads std::threads.  Each index is handled by exactly one
// thread, so results do not depend on nthreads.
template <typename Body>
void parallel_range(int64_t count, int nthreads, Body body) {
    int64_t t = nthreads > 1 ? nthreads : 1;
    if (t > count) t = count > 0 ? count : 1;
    if (t == 1) {
        for (int64_t i = 0; i < count; ++i) body(i);
        return;
    }
    std::vector<std::thread> pool;
    for (int64_t j = 0; j < t; ++j) {
        const int64_t lo = count * j / t, hi = count * (j + 1) / t;
        pool.emplace_back([lo, hi, &body] {
            for (int64_t i = lo; i < hi; ++i) body(i);
        });
    }
    for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

int ref_output_dims(const ref_problem* p, int* Ho, int* Wo) {
    if (!valid(p) || !Ho || !Wo) return -1;
    return out_dims(p, Ho, Wo);
}

int ref_num_points(const ref_problem* p) {
    if (!p) return -1;
    return p->kh * p->kw - (p->remove_center ? 1 : 0);
}

// The weights of the K points of one (pixel, group): the masks, or (softmax
// variant) their softmax over k, exp(m_k - max) / sum_j exp(m_j - max).
std::vector<double> point_weights(const ref_problem* p, const void* offset_mask, int64_t om, int K) {
    std::vector<double> a(K);
    for (int k = 0; k < K; ++k) a[k] = load(offset_mask, p->dtype, om + 2 * K + k);
    if (p->softmax) {
        double mx = a[0];
        for (int k = 1; k < K; ++k) mx = std::max(mx, a[k]);
        double sum = 0.0;
        for (int k = 0; k < K; ++k) {
            a[k] = std::exp(a[k] - mx);
            sum += a[k];
        }
        for (int k = 0; k < K; ++k) a[k] /= sum;
    }
    return a;
}

void ref_encode(int dtype, const double* src, void* dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) store(dst, dtype, i, src[i]);
}

int ref_linear(int64_t M, int Cin, int Cout, int dtype, const void* x, const void* weight,
               const void* bias, void* out) {
    if (M < 0 || Cin < 1 || Cout < 1 || dtype < REF_F32 || dtype > REF_F64 || !x || !weight || !out) return -1;
    for (int64_t m = 0; m < M; ++m) {
        for (int j = 0; j < Cout; ++j) {
            double acc = 0.0;
            for (int c = 0; c < Cin; ++c)
                acc += load(x, dtype, m * Cin + c) * load(weight, dtype, static_cast<int64_t>(j) * Cin + c);
            if (bias) acc += load(bias, dtype, j);
            store(out, dtype, m * Cout + j, acc);
        }
    }
    return 0;
}

int ref_linear_backward(int64_t M, int Cin, int Cout, int dtype, const void* x, const void* weight, const void* g,
                        double* grad_x, double* grad_w, double* grad_b, int nthreads) {
    if (M < 0 || Cin < 1 || Cout < 1 || dtype < REF_F32 || dtype > REF_F64 || (M > 0 && !g)) return -1;
    if ((grad_x && !weight) || (grad_w && !x)) return -1;
    if (grad_x)
        parallel_range(M, nthreads, [&](int64_t m) {
            for (int c = 0; c < Cin; ++c) {
                double acc = 0.0;
                for (int j = 0; j < Cout; ++j)
                    acc += load(g, dtype, m * Cout + j) * load(weight, dtype, static_cast<int64_t>(j) * Cin + c);
                grad_x[m * Cin + c] = acc;
            }
        });
    // For each row j of the weight, one pass over the rows m (in order) keeps the
    // Cin sums of grad_w[j, :] and the sum of grad_b[j] side by side.
    if (grad_w || grad_b)
        parallel_range(Cout, nthreads, [&](int64_t j) {
            std::vector<double> acc(Cin, 0.0);
            double bsum = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                const double gj = load(g, dtype, m * Cout + j);
                bsum += gj;
                if (grad_w)
                    for (int c = 0; c < Cin; ++c) acc[c] += gj * load(x, dtype, m * Cin + c);
            }
            if (grad_w)
                for (int c = 0; c < Cin; ++c) grad_w[j * Cin + c] = acc[c];
            if (grad_b) grad_b[j] = bsum;
        });
    return 0;
}

void ref_decode(int dtype, const void* src, double* dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] = load(src, dtype, i);
}

int ref_forward(const ref_problem* p, const void* value, const void* offset_mask, double* out,
                int nthreads) {
    if (!valid(p) || !value || !offset_mask || !out) return -1;
    int Ho, Wo;
    if (out_dims(p, &Ho, &Wo) != 0) return -1;
    const std::vector<Cell> cells = grid_cells(p);
    const int K = static_cast<int>(cells.size());
    const int C = p->G * p->Cg;
    const int64_t rows = static_cast<int64_t>(p->N) * Ho;
    parallel_range(rows, nthreads, [&](int64_t r) {
        const int n = static_cast<int>(r / Ho);
        const int ho = static_cast<int>(r % Ho);
        for (int wo = 0; wo < Wo; ++wo) {
            const int64_t pix = (static_cast<int64_t>(n) * Ho + ho) * Wo + wo;
            for (int g = 0; g < p->G; ++g) {
                const int64_t om = pix * p->P + static_cast<int64_t>(g) * 3 * K;
                const std::vector<double> a = point_weights(p, offset_mask, om, K);
                for (int c = 0; c < p->Cg; ++c) {
                    double y = 0.0;
                    for (int k = 0; k < K; ++k) {
                        const double dx = load(offset_mask, p->dtype, om + 2 * k);
                        const double dy = load(offset_mask, p->dtype, om + 2 * k + 1);
                        const double m = a[k];
                        double h, w;
                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);
                        const Bilinear b = bilinear_cell(p, h, w);
                        y += m * sample_value(p, value, n, g, c, b);
                    }
                    out[pix * C + static_cast<int64_t>(g) * p->Cg + c] = y;
                }
            }
        }
    });
    return 0;
}

int ref_backward(const ref_problem* p, const void* value, const void* offset_mask,
                 const void* grad_out, double* grad_value, double* grad_offset_mask,
                 int nthreads) {
    if (!valid(p) || !value || !offset_mask || !grad_out || !grad_value || !grad_offset_mask)
        return -1;
    int Ho, Wo;
    if (out_dims(p, &Ho, &Wo) != 0) return -1;
    const std::vector<Cell> cells = grid_cells(p);
    const int K = static_cast<int>(cells.size());
    const int C = p->G * p->Cg;
    const double s = p->location_fp32 ? static_cast<double>(static_cast<float>(p->offset_scale))
                                      : p->offset_scale;
    parallel_range(p->N, nthreads, [&](int64_t n64) {
        const int n = static_cast<int>(n64);
        // grad_value of image n depends only on image n: clear it, then add
        // every sample's contribution in (ho, wo, g, k, corner, c) order.
        const int64_t img = static_cast<int64_t>(p->H) * p->W * C;
        for (int64_t i = 0; i < img; ++i) grad_value[static_cast<int64_t>(n) * img + i] = 0.0;
        for (int ho = 0; ho < Ho; ++ho) {
            for (int wo = 0; wo < Wo; ++wo) {
                const int64_t pix = (static_cast<int64_t>(n) * Ho + ho) * Wo + wo;
                double* gom = grad_offset_mask + pix * p->P;
                for (int e = 0; e < p->P; ++e) gom[e] = 0.0;  // includes the padding tail
                for (int g = 0; g < p->G; ++g) {
                    const int64_t om = pix * p->P + static_cast<int64_t>(g) * 3 * K;
                    const std::vector<double> a = point_weights(p, offset_mask, om, K);
                    std::vector<double> gw(K, 0.0);  // d loss / d (weight of point k) = <gy, S_k>
                    for (int k = 0; k < K; ++k) {
                        const double dx = load(offset_mask, p->dtype, om + 2 * k);
                        const double dy = load(offset_mask, p->dtype, om + 2 * k + 1);
                        const double m = a[k];
                        double h, w;
                        sample_location(p, ho, wo, cells[k], dx, dy, &h, &w);
                        const Bilinear b = bilinear_cell(p, h, w);
                        if (!b.any) continue;  // no pixel touched: S_k = 0, offset gradients 0
                        // Corner values v_ab and the upstream gradient gy, per channel.
                        double gmask = 0.0, gdw = 0.0, gdh = 0.0;
                        for (int c = 0; c < p->Cg; ++c) {
                            const double gy = load(grad_out, p->dtype, pix * C + static_cast<int64_t>(g) * p->Cg + c);
                            double v[2][2];
                            for (int a = 0; a < 2; ++a)
                                for (int bb = 0; bb < 2; ++bb) {
                                    const int y = b.h0 + a, x = b.w0 + bb;
                                    v[a][bb] = inside(p, y, x)
                                                   ? load(value, p->dtype, value_index(p, n, y, x, g, c))
                                                   : 0.0;
                                }
                            // S = bilinear sample; dS/dw and dS/dh inside the floor cell.
                            const double S = (1 - b.lh) * (1 - b.lw) * v[0][0] + (1 - b.lh) * b.lw * v[0][1] +
                                             b.lh * (1 - b.lw) * v[1][0] + b.lh * b.lw * v[1][1];
                            const double dS_dw = (1 - b.lh) * (v[0][1] - v[0][0]) + b.lh * (v[1][1] - v[1][0]);
                            const double dS_dh = (1 - b.lw) * (v[1][0] - v[0][0]) + b.lw * (v[1][1] - v[0][1]);
                            gmask += gy * S;
                            gdw += gy * dS_dw;
                            gdh += gy * dS_dh;
                            // y += m * S: scatter m * weight * gy into each in-image corner.
                            for (int a = 0; a < 2; ++a)
                                for (int bb = 0; bb < 2; ++bb) {
                                    const int y = b.h0 + a, x = b.w0 + bb;
                                    if (!inside(p, y, x)) continue;
                                    const double wt = (a ? b.lh : 1 - b.lh) * (bb ? b.lw : 1 - b.lw);
                                    grad_value[value_index(p, n, y, x, g, c)] += m * wt * gy;
                                }
                        }
                        // location = base + s * offset, so d/d offset = s * m * dS/d location.
                        gom[static_cast<int64_t>(g) * 3 * K + 2 * k] = s * m * gdw;
                        gom[static_cast<int64_t>(g) * 3 * K + 2 * k + 1] = s * m * gdh;
                        gw[k] = gmask;
                    }
                    // Mask gradient: the weight gradient itself, or through the softmax,
                    // d/d m_j = a_j * (gw_j - sum_k a_k gw_k).
                    double dot = 0.0;
                    if (p->softmax)
                        for (int k = 0; k < K; ++k) dot += a[k] * gw[k];
                    for (int k = 0; k < K; ++k)
                        gom[static_cast<int64_t>(g) * 3 * K + 2 * K + k] = p->softmax ? a[k] * (gw[k] - dot) : gw[k];
                }
            }
        }
    });
    return 0;
}

// ---------------------------------------------------------------------------
// Deformable attention (single scale): see dcn4_ref.h.
// ---------------------------------------------------------------------------

static bool attn_valid(const ref_attn_problem* p) {
    if (!p) return false;
    if (p->N < 0 || p->H <= 0 || p->W <= 0 || p->G <= 0 || p->Cg <= 0 || p->Nq < 0 || p->K <= 0) return false;
    if (p->dtype < REF_F32 || p->dtype > REF_F64) return false;
    return p->P >= p->G * 3 * p->K;
}

// The sampling location of one point: reference point + offset_scale * offset.
static void attn_location(const ref_attn_problem* p, float rx, float ry, double dx, double dy, double* h,
                          double* w) {
    if (p->location_fp32) {
        const float s = static_cast<float>(p->offset_scale);
        *h = static_cast<double>(std::fmaf(s, static_cast<float>(dy), ry));
        *w = static_cast<double>(std::fmaf(s, static_cast<float>(dx), rx));
    } else {
        *h = static_cast<double>(ry) + p->offset_scale * dy;
        *w = static_cast<double>(rx) + p->offset_scale * dx;
    }
}

// Corner (y, x) of group g, channel c of image n; 0 outside the image.
static double attn_pixel(const ref_attn_problem* p, const void* value, int n, int y, int x, int g, int c) {
    if (y < 0 || y >= p->H || x < 0 || x >= p->W) return 0.0;
    const int64_t C = static_cast<int64_t>(p->G) * p->Cg;
    return load(value, p->dtype, ((static_cast<int64_t>(n) * p->H + y) * p->W + x) * C + static_cast<int64_t>(g) * p->Cg + c);
}

// Softmax of the K logits of one (query, group), the largest subtracted first.
static std::vector<double> attn_weights(const ref_attn_problem* p, const void* offset_logits, int64_t row) {
    std::vector<double> a(p->K);
    for (int k = 0; k < p->K; ++k) a[k] = load(offset_logits, p->dtype, row + 2 * p->K + k);
    double mx = a[0];
    for (int k = 1; k < p->K; ++k) mx = std::max(mx, a[k]);
    double sum = 0.0;
    for (int k = 0; k < p->K; ++k) {
        a[k] = std::exp(a[k] - mx);
        sum += a[k];
    }
    for (int k = 0; k < p->K; ++k) a[k] /= sum;
    return a;
}

int ref_attn_forward(const ref_attn_problem* p, const void* value, const float* ref_points,
                     const void* offset_logits, double* out, int nthreads) {
    if (!attn_valid(p) || !value || !ref_points || !offset_logits || !out) return -1;
    const int64_t C = static_cast<int64_t>(p->G) * p->Cg;
    parallel_range(static_cast<int64_t>(p->N) * p->Nq, nthreads, [&](int64_t nq) {
        const int n = static_cast<int>(nq / (p->Nq > 0 ? p->Nq : 1));
        const float rx = ref_points[2 * nq], ry = ref_points[2 * nq + 1];
        for (int g = 0; g < p->G; ++g) {
            const int64_t row = nq * p->P + static_cast<int64_t>(g) * 3 * p->K;
            const std::vector<double> a = attn_weights(p, offset_logits, row);
            for (int c = 0; c < p->Cg; ++c) {
                double y = 0.0;
                for (int k = 0; k < p->K; ++k) {
                    double h, w;
                    attn_location(p, rx, ry, load(offset_logits, p->dtype, row + 2 * k),
                                  load(offset_logits, p->dtype, row + 2 * k + 1), &h, &w);
                    // bilinear sample of the zero-extended image: nothing touched beyond [-1, H) x [-1, W)
                    if (!(h >= -1.0 && h < p->H && w >= -1.0 && w < p->W)) continue;
                    const double fh = std::floor(h), fw = std::floor(w);
                    const int h0 = static_cast<int>(fh), w0 = static_cast<int>(fw);
                    const double lh = h - fh, lw = w - fw;
                    double smp = 0.0;
                    for (int a2 = 0; a2 < 2; ++a2)
                        for (int b2 = 0; b2 < 2; ++b2)
                            smp += (a2 ? lh : 1.0 - lh) * (b2 ? lw : 1.0 - lw) *
                                   attn_pixel(p, value, n, h0 + a2, w0 + b2, g, c);
                    y += a[k] * smp;
                }
                out[nq * C + static_cast<int64_t>(g) * p->Cg + c] = y;
            }
        }
    });
    return 0;
}

int ref_attn_backward(const ref_attn_problem* p, const void* value, const float* ref_points,
                      const void* offset_logits, const void* grad_out, double* grad_value,
                      double* grad_offset_logits, int nthreads) {
    if (!attn_valid(p) || !value || !ref_points || !offset_logits || !grad_out || !grad_value ||
        !grad_offset_logits)
        return -1;
    const int64_t C = static_cast<int64_t>(p->G) * p->Cg;
    const int K = p->K;
    const double s = p->location_fp32 ? static_cast<double>(static_cast<float>(p->offset_scale)) : p->offset_scale;
    parallel_range(p->N, nthreads, [&](int64_t n64) {
        const int n = static_cast<int>(n64);
        const int64_t img = static_cast<int64_t>(p->H) * p->W * C;
        for (int64_t i = 0; i < img; ++i) grad_value[n64 * img + i] = 0.0;
        for (int q = 0; q < p->Nq; ++q) {
            const int64_t nq = n64 * p->Nq + q;
            const float rx = ref_points[2 * nq], ry = ref_points[2 * nq + 1];
            double* gol = grad_offset_logits + nq * p->P;
            for (int e = 0; e < p->P; ++e) gol[e] = 0.0;
            for (int g = 0; g < p->G; ++g) {
                const int64_t row = nq * p->P + static_cast<int64_t>(g) * 3 * K;
                const std::vector<double> a = attn_weights(p, offset_logits, row);
                std::vector<double> gw(K, 0.0);  // <gy, S_k>
                for (int k = 0; k < K; ++k) {
                    double h, w;
                    attn_location(p, rx, ry, load(offset_logits, p->dtype, row + 2 * k),
                                  load(offset_logits, p->dtype, row + 2 * k + 1), &h, &w);
                    if (!(h >= -1.0 && h < p->H && w >= -1.0 && w < p->W)) continue;
                    const double fh = std::floor(h), fw = std::floor(w);
                    const int h0 = static_cast<int>(fh), w0 = static_cast<int>(fw);
                    const double lh = h - fh, lw = w - fw;
                    double gS = 0.0, gdw = 0.0, gdh = 0.0;
                    for (int c = 0; c < p->Cg; ++c) {
                        const double gy = load(grad_out, p->dtype, nq * C + static_cast<int64_t>(g) * p->Cg + c);
                        double v[2][2];
                        for (int a2 = 0; a2 < 2; ++a2)
                            for (int b2 = 0; b2 < 2; ++b2) v[a2][b2] = attn_pixel(p, value, n, h0 + a2, w0 + b2, g, c);
                        const double S = (1 - lh) * (1 - lw) * v[0][0] + (1 - lh) * lw * v[0][1] +
                                         lh * (1 - lw) * v[1][0] + lh * lw * v[1][1];
                        gS += gy * S;
                        gdw += gy * ((1 - lh) * (v[0][1] - v[0][0]) + lh * (v[1][1] - v[1][0]));
                        gdh += gy * ((1 - lw) * (v[1][0] - v[0][0]) + lw * (v[1][1] - v[0][1]));
                        for (int a2 = 0; a2 < 2; ++a2)
                            for (int b2 = 0; b2 < 2; ++b2) {
                                const int y = h0 + a2, x = w0 + b2;
                                if (y < 0 || y >= p->H || x < 0 || x >= p->W) continue;
                                const double wt = (a2 ? lh : 1 - lh) * (b2 ? lw : 1 - lw);
                                grad_value[((n64 * p->H + y) * p->W + x) * C + static_cast<int64_t>(g) * p->Cg + c] +=
                                    a[k] * wt * gy;
                            }
                    }
                    gol[static_cast<int64_t>(g) * 3 * K + 2 * k] = s * a[k] * gdw;
                    gol[static_cast<int64_t>(g) * 3 * K + 2 * k + 1] = s * a[k] * gdh;
                    gw[k] = gS;
                }
                double dot = 0.0;
                for (int k = 0; k < K; ++k) dot += a[k] * gw[k];
                for (int k = 0; k < K; ++k) gol[static_cast<int64_t>(g) * 3 * K + 2 * K + k] = a[k] * (gw[k] - dot);
            }
        }
    });
    return 0;
}

}  // extern "C"
