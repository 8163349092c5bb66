// dcn4_api.cu — the C ABI of libdcn4 (declared in include/dcn4.h).
//
// Host side only: validates a call completely before anything reaches the GPU,
// derives the launch geometry from the shape (no tuning tables), and launches
// the kernels of dcn4_forward.cu / dcn4_backward.cu on the caller's stream.
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include <algorithm>

#include "dcn4.h"
#include "dcn4_common.cuh"

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

int elem_bytes(int dtype) { return dtype == DCN4_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Threads of one CTA aim at 256: enough warps per SM to hide gather latency
// while keeping each CTA's offset_mask rows small in shared memory.
constexpr int kTargetThreads = 256;
constexpr size_t kSmemDefault = 48 * 1024;
constexpr size_t kSmemMax = 227 * 1024;
// grad_value pass: 256 threads per CTA and two CTAs per SM, so each CTA's
// bins, candidate list and sample records share this shared-memory budget.
constexpr int kValueThreads = 256;
constexpr size_t kValueSmem = 112 * 1024;
constexpr int kValueMaxBH = 16;    // input rows per tile at most
constexpr int kValueMaxGK = 512;   // groups x points at most
// grad_offset_mask pass: shared memory at most for its offset_mask tiles plus
// the staging of the records it files (beyond it the grad_value pass rescans,
// which for large grids costs far more than the CTAs per SM the staging takes).
constexpr size_t kFileSmem = 200 * 1024;
// Static shared memory of the grad_offset_mask kernel (per-pixel boxes and the
// filing counters), an upper bound.
constexpr size_t kSamplesStaticSmem = 8 * 1024;

// Validates p and fills the kernel geometry.  Touches no GPU state.
// wide: the gathered and stored tensors are 32-byte aligned, so a thread may
// move a 32-byte channel slice with one 256-bit access.
int make_geometry(const dcn4_params* p, bool backward, bool wide, dcn4::Geometry* g, bool full_tiles = false) {
    if (!p) return fail(DCN4_ERR_NULL, "params is NULL");
    if (p->dtype != DCN4_F32 && p->dtype != DCN4_F16 && p->dtype != DCN4_BF16)
        return fail(DCN4_ERR_DTYPE, "dtype %d is not a dcn4_dtype", p->dtype);
    if (p->N < 0 || p->H < 1 || p->W < 1 || p->G < 1 || p->Cg < 1)
        return fail(DCN4_ERR_BAD_SHAPE, "need N >= 0 and H, W, G, Cg >= 1 (got N=%d H=%d W=%d G=%d Cg=%d)", p->N, p->H,
                    p->W, p->G, p->Cg);
    if (p->kh < 1 || p->kw < 1 || p->sh < 1 || p->sw < 1 || p->dh < 1 || p->dw < 1 || p->ph < 0 || p->pw < 0)
        return fail(DCN4_ERR_BAD_SHAPE, "need kernel, stride, dilation >= 1 and padding >= 0");
    if (p->remove_center != 0 && p->remove_center != 1)
        return fail(DCN4_ERR_BAD_SHAPE, "remove_center must be 0 or 1");
    if (p->softmax != 0 && p->softmax != 1) return fail(DCN4_ERR_BAD_SHAPE, "softmax must be 0 or 1");
    if (p->remove_center && (p->kh % 2 == 0 || p->kw % 2 == 0))
        return fail(DCN4_ERR_BAD_SHAPE, "remove_center needs odd kh and kw");
    if (!std::isfinite(p->offset_scale)) return fail(DCN4_ERR_BAD_SHAPE, "offset_scale is not finite");
    if (static_cast<long long>(p->kh) * p->kw > 1024) return fail(DCN4_ERR_UNSUPPORTED, "kh*kw > 1024");
    const int K = p->kh * p->kw - p->remove_center;
    if (K < 1) return fail(DCN4_ERR_BAD_SHAPE, "no sampling point left");
    const long long body = 3LL * p->G * K;
    if (body > (1LL << 30) || p->P < body || p->P % 8 != 0)
        return fail(DCN4_ERR_BAD_P, "P=%d must be a multiple of 8 and >= G*3K=%lld", p->P, body);
    const long long eff_h = static_cast<long long>(p->dh) * (p->kh - 1) + 1;
    const long long eff_w = static_cast<long long>(p->dw) * (p->kw - 1) + 1;
    const long long num_h = p->H + 2LL * p->ph - eff_h, num_w = p->W + 2LL * p->pw - eff_w;
    if (num_h < 0 || num_w < 0) return fail(DCN4_ERR_BAD_SHAPE, "the kernel grid does not fit the padded input");
    const long long Ho = num_h / p->sh + 1, Wo = num_w / p->sw + 1;
    if (p->H >= (1 << 24) || p->W >= (1 << 24) || Ho >= (1 << 24) || Wo >= (1 << 24))
        return fail(DCN4_ERR_UNSUPPORTED, "H, W, Ho, Wo must be < 2^24");
    if (p->ph >= (1 << 24) || p->pw >= (1 << 24) || eff_h >= (1 << 24) || eff_w >= (1 << 24) ||
        static_cast<long long>(p->sh) * Ho >= (1 << 24) || static_cast<long long>(p->sw) * Wo >= (1 << 24))
        return fail(DCN4_ERR_UNSUPPORTED, "grid coordinates must stay below 2^24");
    const long long C = static_cast<long long>(p->G) * p->Cg;
    if (static_cast<long long>(p->H) * p->W * C >= (1LL << 31))
        return fail(DCN4_ERR_UNSUPPORTED, "H*W*C must be < 2^31 per image");
    const int eb = elem_bytes(p->dtype);
    const long long slice_bytes = static_cast<long long>(p->Cg) * eb;
    if (slice_bytes % 16 != 0)
        return fail(DCN4_ERR_UNSUPPORTED, "Cg*sizeof(dtype)=%lld must be a multiple of 16 bytes", slice_bytes);
    const long long vec = (wide && slice_bytes % 32 == 0) ? 2 : 1;
    const long long nslice = slice_bytes / (16 * vec);
    if (nslice > 32 || (nslice & (nslice - 1)) != 0)
        return fail(DCN4_ERR_UNSUPPORTED, "Cg*sizeof(dtype)/32 must be a power of two <= 32 (Cg=%d)", p->Cg);
    const long long lanes_pp = p->G * nslice;
    if (lanes_pp > kTargetThreads)
        return fail(DCN4_ERR_UNSUPPORTED, "G * slices per group = %lld exceeds %d threads", lanes_pp, kTargetThreads);
    const long long total_pix = static_cast<long long>(p->N) * Ho * Wo;
    if (Ho * Wo >= (1LL << 31)) return fail(DCN4_ERR_UNSUPPORTED, "Ho*Wo must be < 2^31");
    if (total_pix > (1LL << 40)) return fail(DCN4_ERR_UNSUPPORTED, "N*Ho*Wo too large");

    // Output pixels per CTA: fill kTargetThreads, then shrink until the
    // shared-memory rows fit the default 48 KB (or, for very long rows, the
    // per-CTA maximum).
    // Shared memory per output pixel: two offset_mask rows (forward: the tiles in
    // flight, a third one only where it still fits three CTAs to an SM; backward:
    // offset_mask and grad_offset_mask rows), and with softmax (forward) its
    // threads' fp32 exponentials.
    const size_t row_bytes = static_cast<size_t>(p->P) * eb * 2 +
                             (p->softmax ? static_cast<size_t>(K) * lanes_pp * sizeof(float) : 0);
    long long ppc = kTargetThreads / lanes_pp;
    while (ppc > 1 && ppc * row_bytes > kSmemDefault) --ppc;
    if (ppc * row_bytes > kSmemMax) return fail(DCN4_ERR_UNSUPPORTED, "P=%d rows do not fit shared memory", p->P);
    if (full_tiles) {  // a power of two of pixels (see below)
        long long q = 1;
        while (q * 2 <= ppc) q *= 2;
        ppc = q;
    }
    // A CTA covers a TH x TW tile of output pixels of one image (TW a power of
    // two, TH = the rest of the pixel budget, both clipped to the image): the
    // shape that leaves the fewest threads idle on the image's ragged edges;
    // among equals the one with more pixels, then the squarer one.  Shapes
    // more than 4:1 are taken only when nothing squarer exists (a 14 x 1 strip
    // fills a 14 x 14 map exactly but gathers from a wider halo per pixel).
    // full_tiles: TH is not clipped to the image, so every tile holds the whole
    // pixel budget (the fused projection's MMA takes N = the tile's pixels).
    long long TW = 1, TH = 1;
    {
        long long best_used = -1, best_slots = 1, best_px = 0, best_skew = 0;
        for (int pass = 0; pass < 2 && best_used < 0; ++pass)
        for (long long tw = 1; tw <= ppc; tw *= 2) {
            if (tw > 1 && tw / 2 >= Wo) break;
            const long long th = full_tiles ? ppc / tw : std::min(ppc / tw, Ho);
            if (pass == 0 && std::max(th, tw) > 4 * std::min(th, tw)) continue;
            const long long slots = (Ho + th - 1) / th * th * ((Wo + tw - 1) / tw * tw);
            const long long used = Ho * Wo;
            const long long px = th * tw, skew = std::max(th, tw) / std::min(th, tw);
            // compare used / slots as fractions without rounding
            const bool better = best_used < 0 || used * best_slots > best_used * slots ||
                                (used * best_slots == best_used * slots &&
                                 (px > best_px || (px == best_px && skew < best_skew)));
            if (better) {
                best_used = used;
                best_slots = slots;
                best_px = px;
                best_skew = skew;
                TW = tw;
                TH = th;
            }
        }
    }
    const long long tiles_h = (Ho + TH - 1) / TH, tiles_w = (Wo + TW - 1) / TW;
    if (static_cast<long long>(p->N) * tiles_h * tiles_w > 0x7fffffffLL)
        return fail(DCN4_ERR_UNSUPPORTED, "grid too large");

    g->N = p->N; g->H = p->H; g->W = p->W; g->G = p->G; g->Cg = p->Cg; g->C = static_cast<int>(C);
    g->Ho = static_cast<int>(Ho); g->Wo = static_cast<int>(Wo); g->P = p->P; g->K = K;
    g->kh = p->kh; g->kw = p->kw; g->sh = p->sh; g->sw = p->sw; g->ph = p->ph; g->pw = p->pw;
    g->dh = p->dh; g->dw = p->dw; g->s = p->offset_scale; g->remove_center = p->remove_center;
    g->softmax = p->softmax;
    g->vec = static_cast<int>(vec);
    g->nslice = static_cast<int>(nslice);
    g->pix_per_cta = static_cast<int>(TH * TW);
    g->total_pix = total_pix;
    g->TH = static_cast<int>(TH);
    g->TW = static_cast<int>(TW);
    g->tiles_h = static_cast<int>(tiles_h);
    g->tiles_w = static_cast<int>(tiles_w);

    // grad_value pass: tiles of BH x BW input pixels.  A strip of LW lanes
    // (one per cell column, BW + 1 of them) covers the tile's width: LW = 32
    // for images at least 16 wide (BW = 31), narrower strips otherwise.
    const long long GK = static_cast<long long>(p->G) * K;
    if (GK > kValueMaxGK) return fail(DCN4_ERR_UNSUPPORTED, "G*K = %lld exceeds %d", GK, kValueMaxGK);
    const int LW = p->W >= 16 ? 32 : p->W >= 8 ? 16 : 8;
    const long long BW = std::min<long long>(p->W, LW - 1);
    const long long brec = eb == 2 ? 8 : 16;
    // Samples per cell per group: K for each output pixel per input pixel.
    const long long dens = K * std::max<long long>(1, (Ho * Wo + static_cast<long long>(p->H) * p->W - 1) /
                                                          (static_cast<long long>(p->H) * p->W));
    g->G = p->G;
    g->K = K;
    g->BW = static_cast<int>(BW);
    g->brec = static_cast<int>(brec);
    // Tallest tile (<= kValueMaxBH rows) whose records fit the budget with a
    // margin over the expected count (records beyond it send the tile to the
    // direct path).
    long long BH = std::min<long long>(kValueMaxBH, p->H);
    for (;; --BH) {
        const long long expect = static_cast<long long>(p->G) * (BH + 1) * (BW + 1) * dens;
        g->BH = static_cast<int>(BH);
        g->bcap = static_cast<int>(std::min<long long>(expect + expect / 16 + 512, 1LL << 24));
        if (dcn4::backward_value_smem_bytes(*g) <= kValueSmem || BH == 1) break;
    }
    if (dcn4::backward_value_smem_bytes(*g) > kValueSmem) {
        g->bcap = 0;
        const size_t fixed = dcn4::backward_value_smem_bytes(*g);
        if (fixed + 1024 * brec > kValueSmem) return fail(DCN4_ERR_UNSUPPORTED, "too many groups for the grad_value tile");
        g->bcap = static_cast<int>((kValueSmem - fixed) / brec);
    }
    // Segments: enough (group, slice, segment) strips for every strip slot of the CTA.
    const long long slots = (kValueThreads / 32) * (32 / LW);
    long long nseg = std::min<long long>(BH, std::max<long long>(1, (slots + lanes_pp - 1) / lanes_pp));
    const long long BS = (BH + nseg - 1) / nseg;
    nseg = (BH + BS - 1) / BS;
    const long long btiles_h = (p->H + BH - 1) / BH, btiles_w = (p->W + BW - 1) / BW;
    if (static_cast<long long>(p->N) * btiles_h * btiles_w > 0x7fffffffLL)
        return fail(DCN4_ERR_UNSUPPORTED, "grid too large");
    g->btiles_h = static_cast<int>(btiles_h);
    g->btiles_w = static_cast<int>(btiles_w);
    g->bthreads = kValueThreads;
    g->LW = LW;
    g->BS = static_cast<int>(BS);
    g->nseg = static_cast<int>(nseg);
    // Buckets for 16-bit dtypes, when a record can name its output pixel as
    // (ho << 16) | wo and its bin in 16 bits.
    const long long nbins = static_cast<long long>(p->G) * (BH + 1) * (BW + 1);
    g->buckets = eb == 2 && Ho <= 65535 && Wo <= 65535 && nbins <= 65535;

    // Filing window (64 grad_value tiles): enough tile rows for the rows a CTA's
    // samples span -- its TH output rows, the grid, and about 8 pixels of
    // offsets either way -- the rest of the 64 as columns.
    {
        const long long span = (TH - 1) * p->sh + static_cast<long long>(p->kh - 1) * p->dh + 2 * 8 + 2;
        const long long need = (span + BH - 1) / BH + 1;
        int wl = 3;  // 8 x 8, and always for 3 x 3 grids, whose kernels are compiled for it
        while (wl > 0 && (64 >> wl) < need && !(p->kh == 3 && p->kw == 3)) --wl;
        g->fwin_wl = wl;
        g->fwin_h = 64 >> wl;
    }
    g->bh_magic = 0xffffffffu / static_cast<uint32_t>(BH) + 1u;  // BH, BW >= 2 use __umulhi; 1 is special-cased
    g->bw_magic = 0xffffffffu / static_cast<uint32_t>(BW) + 1u;
    // ... and when the grad_offset_mask CTA can stage its records in shared memory.
    if (g->buckets && (dcn4::backward_smem_bytes(*g, eb) > kFileSmem ||
                       static_cast<long long>(dcn4::filing_chunk(*g)) * dcn4::samples_threads(*g) > (1 << 13)))
        g->buckets = 0;
    // The grad_offset_mask CTA's dynamic shared memory, next to its static arrays.
    if (backward && dcn4::backward_smem_bytes(*g, eb) + kSamplesStaticSmem > kSmemMax)
        return fail(DCN4_ERR_UNSUPPORTED, "the backward's rows of P=%d (K=%d) do not fit shared memory", p->P, K);
    return DCN4_OK;
}

// Backward workspace, each part starting on a 256-byte boundary.  The header
// (zeroed by one memset per call): kDiagWords fallback counters, one reach word
// per image (stored as R + 1, 0: no sample touches the image), and for 16-bit
// dtypes with buckets one record counter per grad_value tile.  Then one cell
// box (4 bytes) per output pixel; then for fp32 a 2-byte cell code per sample,
// for 16-bit dtypes (with buckets) each tile's bucket of bcap records: 4-byte
// output pixels, then 8-byte bin, mask bits and fractions.
size_t round256(size_t b) { return (b + 255) / 256 * 256; }
size_t num_value_tiles(const dcn4::Geometry& g) { return static_cast<size_t>(g.N) * g.btiles_h * g.btiles_w; }
size_t header_words(const dcn4::Geometry& g, int dtype) {
    return dcn4::kDiagWords + static_cast<size_t>(g.N) + (dtype != DCN4_F32 && g.buckets ? num_value_tiles(g) : 0);
}
size_t header_bytes(const dcn4::Geometry& g, int dtype) { return round256(header_words(g, dtype) * sizeof(int)); }
size_t box_bytes(const dcn4::Geometry& g) { return round256(static_cast<size_t>(g.total_pix) * 4); }
size_t num_samples(const dcn4::Geometry& g) { return static_cast<size_t>(g.total_pix) * g.G * g.K; }
size_t workspace_bytes(const dcn4::Geometry& g, int dtype) {
    size_t b = header_bytes(g, dtype) + box_bytes(g);
    if (dtype == DCN4_F32) return b + round256(num_samples(g) * 2);
    if (!g.buckets) return b;
    const size_t recs = num_value_tiles(g) * static_cast<size_t>(g.bcap);
    return b + round256(recs * 4) + recs * 8;
}
int* reach_words(void* workspace) { return static_cast<int*>(workspace) + dcn4::kDiagWords; }
uint32_t* box_words(const dcn4::Geometry& g, int dtype, void* workspace) {
    return reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + header_bytes(g, dtype));
}
dcn4::SampleArrays sample_arrays(const dcn4::Geometry& g, int dtype, const void* workspace) {
    char* ws = static_cast<char*>(const_cast<void*>(workspace));
    char* base = ws + header_bytes(g, dtype) + box_bytes(g);
    dcn4::SampleArrays sa = {};
    sa.diag = reinterpret_cast<int*>(ws);
    if (dtype == DCN4_F32) {
        sa.code = reinterpret_cast<uint16_t*>(base);
    } else if (g.buckets) {
        const size_t recs = num_value_tiles(g) * static_cast<size_t>(g.bcap);
        sa.tile_count = reach_words(ws) + g.N;
        sa.bucket_pix = reinterpret_cast<uint32_t*>(base);
        sa.bucket_rec = reinterpret_cast<uint64_t*>(base + round256(recs * 4));
    }
    return sa;
}

// Validates a deformable attention call and fills the kernel geometry (value
// map, points per query, row length, slices).  Touches no GPU state.
int make_attn_geometry(const dcn4_attn_params* p, bool wide, dcn4::Geometry* g) {
    if (!p) return fail(DCN4_ERR_NULL, "params is NULL");
    if (p->dtype != DCN4_F32 && p->dtype != DCN4_F16 && p->dtype != DCN4_BF16)
        return fail(DCN4_ERR_DTYPE, "dtype %d is not a dcn4_dtype", p->dtype);
    if (p->N < 0 || p->H < 1 || p->W < 1 || p->G < 1 || p->Cg < 1 || p->Nq < 0 || p->K < 1)
        return fail(DCN4_ERR_BAD_SHAPE, "need N, Nq >= 0 and H, W, G, Cg, K >= 1");
    if (!std::isfinite(p->offset_scale)) return fail(DCN4_ERR_BAD_SHAPE, "offset_scale is not finite");
    if (p->K > 1024) return fail(DCN4_ERR_UNSUPPORTED, "K > 1024");
    const long long body = 3LL * p->G * p->K;
    if (body > (1LL << 30) || p->P < body || p->P % 8 != 0)
        return fail(DCN4_ERR_BAD_P, "P=%d must be a multiple of 8 and >= G*3K=%lld", p->P, body);
    if (p->H >= (1 << 24) || p->W >= (1 << 24)) return fail(DCN4_ERR_UNSUPPORTED, "H, W must be < 2^24");
    const long long C = static_cast<long long>(p->G) * p->Cg;
    if (static_cast<long long>(p->H) * p->W * C >= (1LL << 31))
        return fail(DCN4_ERR_UNSUPPORTED, "H*W*C must be < 2^31 per image");
    const int eb = elem_bytes(p->dtype);
    const long long slice_bytes = static_cast<long long>(p->Cg) * eb;
    if (slice_bytes % 16 != 0)
        return fail(DCN4_ERR_UNSUPPORTED, "Cg*sizeof(dtype)=%lld must be a multiple of 16 bytes", slice_bytes);
    const long long vec = (wide && slice_bytes % 32 == 0) ? 2 : 1;
    const long long nslice = slice_bytes / (16 * vec);
    if (nslice > 32 || (nslice & (nslice - 1)) != 0)
        return fail(DCN4_ERR_UNSUPPORTED, "Cg*sizeof(dtype)/32 must be a power of two <= 32 (Cg=%d)", p->Cg);
    if (p->G * nslice > kTargetThreads)
        return fail(DCN4_ERR_UNSUPPORTED, "G * slices per group = %lld exceeds %d threads", p->G * nslice, kTargetThreads);
    const long long queries = static_cast<long long>(p->N) * p->Nq;
    if (queries > (1LL << 40)) return fail(DCN4_ERR_UNSUPPORTED, "N*Nq too large");
    *g = dcn4::Geometry{};
    g->N = p->N; g->H = p->H; g->W = p->W; g->G = p->G; g->Cg = p->Cg; g->C = static_cast<int>(C);
    g->K = p->K; g->P = p->P; g->s = p->offset_scale; g->softmax = 1;
    g->vec = static_cast<int>(vec);
    g->nslice = static_cast<int>(nslice);
    g->Ho = 1; g->Wo = 1;
    if (dcn4::attn_smem_bytes(*g, eb, true) > kSmemMax)
        return fail(DCN4_ERR_UNSUPPORTED, "K=%d points and P=%d rows do not fit shared memory", p->K, p->P);
    const long long qb = std::max(1LL, static_cast<long long>(kTargetThreads) / (p->G * nslice));
    if ((queries + qb - 1) / qb > 0x7fffffffLL) return fail(DCN4_ERR_UNSUPPORTED, "grid too large");
    return DCN4_OK;
}

}  // namespace

extern "C" {

int dcn4_version(void) { return DCN4_VERSION; }

int dcn4_num_points(const dcn4_params* p) {
    if (!p) return fail(DCN4_ERR_NULL, "params is NULL");
    if (p->kh < 1 || p->kw < 1 || (p->remove_center != 0 && p->remove_center != 1))
        return fail(DCN4_ERR_BAD_SHAPE, "bad kernel size or remove_center");
    const int K = p->kh * p->kw - p->remove_center;
    return K >= 1 ? K : fail(DCN4_ERR_BAD_SHAPE, "no sampling point left");
}

int dcn4_padded_offset_dim(int G, int K) {
    if (G < 1 || K < 1 || static_cast<long long>(G) * K > (1LL << 28))
        return fail(DCN4_ERR_BAD_SHAPE, "need G >= 1 and K >= 1");
    return (G * 3 * K + 7) / 8 * 8;
}

int dcn4_output_dims(const dcn4_params* p, int* Ho, int* Wo) {
    if (!Ho || !Wo) return fail(DCN4_ERR_NULL, "Ho/Wo is NULL");
    dcn4::Geometry g;
    const int st = make_geometry(p, false, true, &g);
    if (st != DCN4_OK) return st;
    *Ho = g.Ho;
    *Wo = g.Wo;
    return DCN4_OK;
}

int dcn4_check_params(const dcn4_params* p) {
    dcn4::Geometry g;
    for (int backward = 0; backward < 2; ++backward)
        for (int wide = 0; wide < 2; ++wide) {
            const int st = make_geometry(p, backward, wide, &g);
            if (st != DCN4_OK) return st;
        }
    return DCN4_OK;
}

int dcn4_forward(const dcn4_params* p, const void* value, const void* offset_mask, void* out, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, false, aligned32(value) && aligned32(out), &g);
    if (st != DCN4_OK) return st;
    if (g.total_pix == 0) return DCN4_OK;
    if (!value || !offset_mask || !out) return fail(DCN4_ERR_NULL, "value, offset_mask and out must be non-NULL");
    if (!aligned16(value) || !aligned16(offset_mask) || !aligned16(out))
        return fail(DCN4_ERR_MISALIGNED, "value, offset_mask and out must be 16-byte aligned");
    const cudaError_t e =
        dcn4::launch_forward(g, p->dtype, value, offset_mask, out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "forward launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

int dcn4_forward_linear(const dcn4_params* p, int Cx, const void* value, const void* x, const void* weight,
                        const void* bias, void* out, void* offset_mask_out, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, false, aligned32(value) && aligned32(out), &g);
    if (st != DCN4_OK) return st;
    if (p->dtype == DCN4_F32) return fail(DCN4_ERR_UNSUPPORTED, "the fused linear producer takes fp16 or bf16");
    if (Cx < 16 || Cx % 16 != 0 || Cx > (1 << 16))
        return fail(DCN4_ERR_BAD_SHAPE, "Cx=%d must be a positive multiple of 16", Cx);
    if (dcn4::forward_linear_smem_bytes(g, Cx, dcn4::forward_linear_mode(g, Cx)) > kSmemMax)
        return fail(DCN4_ERR_UNSUPPORTED, "x rows of Cx=%d with P=%d do not fit shared memory", Cx, p->P);
    if (static_cast<long long>(g.Ho) * g.Wo * Cx >= (1LL << 31) || static_cast<long long>(p->P) * Cx >= (1LL << 31))
        return fail(DCN4_ERR_UNSUPPORTED, "x or weight too large");
    if (g.total_pix == 0) return DCN4_OK;
    if (!value || !x || !weight || !out) return fail(DCN4_ERR_NULL, "value, x, weight and out must be non-NULL");
    if (!aligned16(value) || !aligned16(x) || !aligned16(weight) || !aligned16(out) || !aligned16(bias) ||
        !aligned16(offset_mask_out))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const cudaError_t e = dcn4::launch_forward_linear(g, p->dtype, value, x, weight, bias, out, offset_mask_out, Cx,
                                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "forward_linear launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

int dcn4_forward_proj(const dcn4_params* p, int Cout, const void* value, const void* offset_mask, const void* weight,
                      const void* bias, void* out, void* core_out, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, false, aligned32(value), &g, true);
    if (st != DCN4_OK) return st;
    if (p->dtype == DCN4_F32) return fail(DCN4_ERR_UNSUPPORTED, "the fused output projection takes fp16 or bf16");
    if (Cout < 16 || Cout % 16 != 0 || Cout > (1 << 16))
        return fail(DCN4_ERR_BAD_SHAPE, "Cout=%d must be a positive multiple of 16", Cout);
    if (Cout > 128) return fail(DCN4_ERR_UNSUPPORTED, "the fused projection forms at most 128 outputs (Cout=%d)", Cout);
    if (!dcn4::forward_proj_shape_ok(g, Cout))
        return fail(DCN4_ERR_UNSUPPORTED,
                    "the fused projection needs C a multiple of 64 up to 256 and 16-, 32- or 64-pixel tiles "
                    "(C=%d, G=%d: %d-pixel tiles)",
                    g.C, p->G, g.pix_per_cta);
    if (dcn4::forward_proj_smem_bytes(g, Cout) > kSmemMax)
        return fail(DCN4_ERR_UNSUPPORTED, "P=%d rows with C=%d do not fit shared memory", p->P, g.C);
    if (g.total_pix == 0) return DCN4_OK;
    if (!value || !offset_mask || !weight || !out)
        return fail(DCN4_ERR_NULL, "value, offset_mask, weight and out must be non-NULL");
    if (!aligned16(value) || !aligned16(offset_mask) || !aligned16(weight) || !aligned16(out) || !aligned16(bias) ||
        !aligned16(core_out))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const cudaError_t e = dcn4::launch_forward_proj(g, p->dtype, value, offset_mask, weight, bias, out, core_out, Cout,
                                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "forward_proj launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

int dcn4_forward_tc_status(int reset) {
    unsigned v = 0u;
    const cudaError_t e = dcn4::forward_tc_status(&v, reset != 0);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "reading the forward status word: %s", cudaGetErrorString(e));
    return static_cast<int>(v & 0x7fffffffu);
}

size_t dcn4_backward_workspace_size(const dcn4_params* p) {
    dcn4::Geometry g;
    if (make_geometry(p, true, true, &g) != DCN4_OK) return 0;
    return workspace_bytes(g, p->dtype);
}

int dcn4_backward_offset_mask(const dcn4_params* p, const void* value, const void* offset_mask, const void* grad_out,
                              void* grad_offset_mask, void* workspace, size_t workspace_bytes, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, true, aligned32(value) && aligned32(grad_out), &g);
    if (st != DCN4_OK) return st;
    if (g.total_pix == 0) return DCN4_OK;
    if (!value || !offset_mask || !grad_out || !grad_offset_mask)
        return fail(DCN4_ERR_NULL, "value, offset_mask, grad_out and grad_offset_mask must be non-NULL");
    if (!aligned16(value) || !aligned16(offset_mask) || !aligned16(grad_out) || !aligned16(grad_offset_mask))
        return fail(DCN4_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
    const size_t need = dcn4_backward_workspace_size(p);
    if (!workspace || workspace_bytes < need)
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    int* reach = reach_words(workspace);
    uint32_t* boxes = box_words(g, p->dtype, workspace);
    const dcn4::SampleArrays sa = sample_arrays(g, p->dtype, workspace);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // counters, reach words and bucket counters: one memset
    cudaError_t e = cudaMemsetAsync(workspace, 0, header_words(g, p->dtype) * sizeof(int), s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "workspace reset: %s", cudaGetErrorString(e));
    e = dcn4::launch_backward_samples(g, p->dtype, value, offset_mask, grad_out, grad_offset_mask, reach, sa, boxes, s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "grad_offset_mask launch: %s", cudaGetErrorString(e));

    return DCN4_OK;
}

int dcn4_backward_value(const dcn4_params* p, const void* offset_mask, const void* grad_out, void* grad_value,
                        const void* workspace, size_t workspace_bytes, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, true, aligned32(grad_out) && aligned32(grad_value), &g);
    if (st != DCN4_OK) return st;
    if (g.total_pix == 0) return DCN4_OK;
    if (!offset_mask || !grad_out || !grad_value)
        return fail(DCN4_ERR_NULL, "offset_mask, grad_out and grad_value must be non-NULL");
    if (!aligned16(offset_mask) || !aligned16(grad_out) || !aligned16(grad_value))
        return fail(DCN4_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
    const size_t need = dcn4_backward_workspace_size(p);
    if (!workspace || workspace_bytes < need)
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const int* reach = reach_words(const_cast<void*>(workspace));
    const uint32_t* boxes = box_words(g, p->dtype, const_cast<void*>(workspace));
    const dcn4::SampleArrays sa = sample_arrays(g, p->dtype, workspace);
    const cudaError_t e = dcn4::launch_backward_value(g, p->dtype, offset_mask, grad_out, grad_value, reach, sa,
                                                      boxes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "grad_value launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

int dcn4_backward(const dcn4_params* p, const void* value, const void* offset_mask, const void* grad_out,
                  void* grad_value, void* grad_offset_mask, void* workspace, size_t workspace_bytes, void* stream) {
    // Check everything the second stage needs before launching the first.
    dcn4::Geometry g;
    const int st = make_geometry(p, true, false, &g);
    if (st != DCN4_OK) return st;
    if (g.total_pix == 0) return DCN4_OK;
    if (!grad_value) return fail(DCN4_ERR_NULL, "grad_value must be non-NULL");
    if (!aligned16(grad_value)) return fail(DCN4_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
    const int a = dcn4_backward_offset_mask(p, value, offset_mask, grad_out, grad_offset_mask, workspace,
                                            workspace_bytes, stream);
    if (a != DCN4_OK) return a;
    return dcn4_backward_value(p, offset_mask, grad_out, grad_value, workspace, workspace_bytes, stream);
}

size_t dcn4_backward_linear_workspace_size(const dcn4_params* p, int Cx) {
    const size_t b = dcn4_backward_workspace_size(p);
    if (b == 0 || Cx < 1 || static_cast<long long>(p->P) * Cx >= (1LL << 31)) return 0;
    return round256(b) + round256(dcn4::linear_backward_workspace_bytes(p->P, Cx));
}

int dcn4_backward_linear(const dcn4_params* p, int Cx, const void* value, const void* offset_mask, const void* x,
                         const void* weight, const void* grad_out, void* grad_value, void* grad_offset_mask,
                         void* grad_x, void* grad_weight, void* grad_bias, void* workspace, size_t workspace_bytes,
                         void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, true, false, &g);
    if (st != DCN4_OK) return st;
    if (p->dtype == DCN4_F32) return fail(DCN4_ERR_UNSUPPORTED, "the linear producer takes fp16 or bf16");
    if (Cx < 16 || Cx % 16 != 0 || Cx > (1 << 16))
        return fail(DCN4_ERR_BAD_SHAPE, "Cx=%d must be a positive multiple of 16", Cx);
    if (static_cast<long long>(p->P) * Cx >= (1LL << 31) || g.total_pix >= (1LL << 31))
        return fail(DCN4_ERR_UNSUPPORTED, "x or weight too large (N*Ho*Wo and P*Cx must be < 2^31)");
    if (!aligned16(x) || !aligned16(weight) || !aligned16(grad_x) || !aligned16(grad_weight) || !aligned16(grad_bias))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const size_t need = dcn4_backward_linear_workspace_size(p, Cx);
    if (!workspace || workspace_bytes < need)
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t eb = static_cast<size_t>(elem_bytes(p->dtype));
    if (g.total_pix == 0) {
        // no output pixels: the weight and bias gradients are empty sums
        cudaError_t e = cudaSuccess;
        if (grad_weight) e = cudaMemsetAsync(grad_weight, 0, static_cast<size_t>(p->P) * Cx * eb, s);
        if (e == cudaSuccess && grad_bias) e = cudaMemsetAsync(grad_bias, 0, static_cast<size_t>(p->P) * eb, s);
        if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "zeroing grad_weight/grad_bias: %s", cudaGetErrorString(e));
        return DCN4_OK;
    }
    if (!grad_offset_mask) return fail(DCN4_ERR_NULL, "grad_offset_mask must be non-NULL");
    if ((grad_x && !weight) || (grad_weight && !x))
        return fail(DCN4_ERR_NULL, "grad_x needs weight and grad_weight needs x");
    const size_t lin_off = round256(dcn4_backward_workspace_size(p));
    const int a = dcn4_backward(p, value, offset_mask, grad_out, grad_value, grad_offset_mask, workspace, lin_off, stream);
    if (a != DCN4_OK) return a;
    float* acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + lin_off);
    const cudaError_t e = dcn4::launch_linear_backward(p->dtype, g.total_pix, p->P, Cx, x, weight, grad_offset_mask,
                                                       grad_x, grad_weight, grad_bias, acc, s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "linear backward launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

size_t dcn4_backward_proj_workspace_size(const dcn4_params* p, int Cout) {
    dcn4::Geometry g;
    if (make_geometry(p, true, true, &g) != DCN4_OK || Cout < 1 || static_cast<long long>(Cout) * g.C >= (1LL << 31))
        return 0;
    const size_t b = dcn4_backward_workspace_size(p);
    if (b == 0) return 0;
    const size_t core = static_cast<size_t>(g.total_pix) * g.C * static_cast<size_t>(elem_bytes(p->dtype));
    return round256(b) + round256(core) + round256(dcn4::linear_backward_workspace_bytes(Cout, g.C));
}

int dcn4_backward_proj(const dcn4_params* p, int Cout, const void* value, const void* offset_mask,
                       const void* core_out, const void* weight, const void* grad_out, void* grad_value,
                       void* grad_offset_mask, void* grad_weight, void* grad_bias, void* workspace,
                       size_t workspace_bytes, void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, true, false, &g);
    if (st != DCN4_OK) return st;
    if (p->dtype == DCN4_F32) return fail(DCN4_ERR_UNSUPPORTED, "the output projection takes fp16 or bf16");
    if (Cout < 16 || Cout % 16 != 0 || Cout > (1 << 16))
        return fail(DCN4_ERR_BAD_SHAPE, "Cout=%d must be a positive multiple of 16", Cout);
    if (g.C % 16 != 0) return fail(DCN4_ERR_BAD_SHAPE, "C=%d must be a multiple of 16", g.C);
    if (static_cast<long long>(Cout) * g.C >= (1LL << 31) || g.total_pix >= (1LL << 31))
        return fail(DCN4_ERR_UNSUPPORTED, "too large (N*Ho*Wo and Cout*C must be < 2^31)");
    if (!aligned16(core_out) || !aligned16(weight) || !aligned16(grad_out) || !aligned16(grad_weight) ||
        !aligned16(grad_bias))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const size_t need = dcn4_backward_proj_workspace_size(p, Cout);
    if (!workspace || workspace_bytes < need)
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t eb = static_cast<size_t>(elem_bytes(p->dtype));
    if (g.total_pix == 0) {
        // no output pixels: the weight and bias gradients are empty sums
        cudaError_t e = cudaSuccess;
        if (grad_weight) e = cudaMemsetAsync(grad_weight, 0, static_cast<size_t>(Cout) * g.C * eb, s);
        if (e == cudaSuccess && grad_bias) e = cudaMemsetAsync(grad_bias, 0, static_cast<size_t>(Cout) * eb, s);
        if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "zeroing grad_weight/grad_bias: %s", cudaGetErrorString(e));
        return DCN4_OK;
    }
    // everything the aggregation's backward checks, before the first launch
    if (!value || !offset_mask || !weight || !grad_out || !grad_value || !grad_offset_mask)
        return fail(DCN4_ERR_NULL,
                    "value, offset_mask, weight, grad_out, grad_value and grad_offset_mask must be non-NULL");
    if (!aligned16(value) || !aligned16(offset_mask) || !aligned16(grad_value) || !aligned16(grad_offset_mask))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    if (grad_weight && !core_out) return fail(DCN4_ERR_NULL, "grad_weight needs core_out");
    // [core backward workspace][grad of the core output, N*Ho*Wo*C][grad_W / grad_b accumulators]
    const size_t core_ws = round256(dcn4_backward_workspace_size(p));
    const size_t gcore_bytes = round256(static_cast<size_t>(g.total_pix) * g.C * eb);
    void* gcore = static_cast<char*>(workspace) + core_ws;
    float* acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + core_ws + gcore_bytes);
    // the projection's gradients first: grad_core = grad_out W (rounded to the dtype, as the
    // unfused pair would store it), grad_W = grad_out^T core_out, grad_b = column sums of grad_out
    const cudaError_t e = dcn4::launch_linear_backward(p->dtype, g.total_pix, Cout, g.C, core_out, weight, grad_out,
                                                       gcore, grad_weight, grad_bias, acc, s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "projection backward launch: %s", cudaGetErrorString(e));
    return dcn4_backward(p, value, offset_mask, gcore, grad_value, grad_offset_mask, workspace, core_ws, stream);
}

int dcn4_attn_check_params(const dcn4_attn_params* p) {
    dcn4::Geometry g;
    for (int wide = 0; wide < 2; ++wide) {
        const int st = make_attn_geometry(p, wide, &g);
        if (st != DCN4_OK) return st;
    }
    return DCN4_OK;
}

int dcn4_attn_forward(const dcn4_attn_params* p, const void* value, const float* ref_points, const void* offset_logits,
                      void* out, void* stream) {
    dcn4::Geometry g;
    const int st = make_attn_geometry(p, aligned32(value) && aligned32(out), &g);
    if (st != DCN4_OK) return st;
    if (static_cast<long long>(p->N) * p->Nq == 0) return DCN4_OK;
    if (!value || !ref_points || !offset_logits || !out)
        return fail(DCN4_ERR_NULL, "value, ref_points, offset_logits and out must be non-NULL");
    if (!aligned16(value) || !aligned16(ref_points) || !aligned16(offset_logits) || !aligned16(out))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const cudaError_t e = dcn4::launch_attn_forward(g, p->dtype, p->Nq, value, ref_points, offset_logits, out,
                                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "attention forward launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

size_t dcn4_attn_backward_workspace_size(const dcn4_attn_params* p) {
    dcn4::Geometry g;
    if (make_attn_geometry(p, true, &g) != DCN4_OK) return 0;
    if (p->dtype == DCN4_F32) return 0;
    return round256(static_cast<size_t>(p->N) * p->H * p->W * g.C * sizeof(float));
}

int dcn4_attn_backward(const dcn4_attn_params* p, const void* value, const float* ref_points, const void* offset_logits,
                       const void* grad_out, void* grad_value, void* grad_offset_logits, void* workspace,
                       size_t workspace_bytes, void* stream) {
    dcn4::Geometry g;
    const int st = make_attn_geometry(p, aligned32(value) && aligned32(grad_out), &g);
    if (st != DCN4_OK) return st;
    if (!grad_value && p->N > 0) return fail(DCN4_ERR_NULL, "grad_value must be non-NULL");
    if (p->N == 0) return DCN4_OK;
    if (!aligned16(grad_value)) return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const size_t need = dcn4_attn_backward_workspace_size(p);
    if (need && (!workspace || workspace_bytes < need))
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (need && !aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const bool any_query = p->Nq > 0;
    if (any_query && (!value || !ref_points || !offset_logits || !grad_out || !grad_offset_logits))
        return fail(DCN4_ERR_NULL, "value, ref_points, offset_logits, grad_out and grad_offset_logits must be non-NULL");
    if (any_query && (!aligned16(value) || !aligned16(ref_points) || !aligned16(offset_logits) ||
                      !aligned16(grad_out) || !aligned16(grad_offset_logits)))
        return fail(DCN4_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t elems = static_cast<size_t>(p->N) * p->H * p->W * g.C;
    float* acc = p->dtype == DCN4_F32 ? static_cast<float*>(grad_value) : static_cast<float*>(workspace);
    cudaError_t e = cudaMemsetAsync(acc, 0, elems * sizeof(float), s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "accumulator reset: %s", cudaGetErrorString(e));
    if (!any_query) {
        // no query samples anything: grad_value is zero (rounded from the cleared accumulator)
        if (p->dtype != DCN4_F32) e = cudaMemsetAsync(grad_value, 0, elems * elem_bytes(p->dtype), s);
        if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "grad_value reset: %s", cudaGetErrorString(e));
        return DCN4_OK;
    }
    e = dcn4::launch_attn_backward(g, p->dtype, p->Nq, value, ref_points, offset_logits, grad_out, grad_value,
                                   grad_offset_logits, acc, s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "attention backward launch: %s", cudaGetErrorString(e));
    return DCN4_OK;
}

int dcn4_backward_diagnostics(const dcn4_params* p, const void* workspace, size_t workspace_bytes, int* counts,
                              void* stream) {
    dcn4::Geometry g;
    const int st = make_geometry(p, true, false, &g);
    if (st != DCN4_OK) return st;
    if (!counts) return fail(DCN4_ERR_NULL, "counts must be non-NULL");
    counts[0] = counts[1] = counts[2] = 0;
    if (g.total_pix == 0) return DCN4_OK;
    const size_t need = dcn4_backward_workspace_size(p);
    if (!workspace || workspace_bytes < need)
        return fail(DCN4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(DCN4_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    int host[dcn4::kDiagWords] = {};
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(host, workspace, sizeof host, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(DCN4_ERR_LAUNCH, "diagnostics read: %s", cudaGetErrorString(e));
    counts[0] = host[dcn4::kDiagCorruptBucket];
    counts[1] = host[dcn4::kDiagRescan];
    counts[2] = host[dcn4::kDiagDirect];
    return DCN4_OK;
}

const char* dcn4_status_string(int status) {
    switch (status) {
        case DCN4_OK: return "DCN4_OK";
        case DCN4_ERR_NULL: return "DCN4_ERR_NULL";
        case DCN4_ERR_BAD_SHAPE: return "DCN4_ERR_BAD_SHAPE";
        case DCN4_ERR_BAD_P: return "DCN4_ERR_BAD_P";
        case DCN4_ERR_MISALIGNED: return "DCN4_ERR_MISALIGNED";
        case DCN4_ERR_UNSUPPORTED: return "DCN4_ERR_UNSUPPORTED";
        case DCN4_ERR_WORKSPACE: return "DCN4_ERR_WORKSPACE";
        case DCN4_ERR_LAUNCH: return "DCN4_ERR_LAUNCH";
        case DCN4_ERR_DTYPE: return "DCN4_ERR_DTYPE";
        default: return "DCN4_UNKNOWN_STATUS";
    }
}

const char* dcn4_last_error(void) { return g_last_error; }

}  // extern "C"
