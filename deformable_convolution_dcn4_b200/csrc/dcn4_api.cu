// dcn4_api.cu -- the C ABI declared in include/dcn4.h: argument validation,
// kernel choice, tiling of the shared-memory halo kernel, TMA descriptor
// encoding and launch. Host code only; every arithmetic step of the operator
// runs in the kernels of dcn4_kernels.cu.
#include <cudaTypedefs.h>
#include <string.h>

#include <limits>
#include <mutex>

#include "dcn4.h"
#include "dcn4_launch.h"

using namespace dcn4;

namespace {

constexpr long long kMaxElems = (1ll << 31) - 1;

bool out_hw(const dcn4_desc &d, int *Ho, int *Wo) {
    if (d.N <= 0 || d.H <= 0 || d.W <= 0 || d.C <= 0 || d.G <= 0) return false;
    if (d.C % d.G != 0 || d.G > kMaxGroups) return false;
    if (d.kh <= 0 || d.kw <= 0 || d.kh * d.kw > 64) return false;
    if (d.stride_h <= 0 || d.stride_w <= 0 || d.dil_h <= 0 || d.dil_w <= 0) return false;
    if (d.pad_h < 0 || d.pad_w < 0) return false;
    const long long ho = ((long long)d.H + 2ll * d.pad_h - (long long)d.dil_h * (d.kh - 1) - 1) / d.stride_h + 1;
    const long long wo = ((long long)d.W + 2ll * d.pad_w - (long long)d.dil_w * (d.kw - 1) - 1) / d.stride_w + 1;
    if (ho <= 0 || wo <= 0 || ho > (1 << 24) || wo > (1 << 24)) return false;
    *Ho = (int)ho;
    *Wo = (int)wo;
    return true;
}

bool make_geometry(const dcn4_desc *d, Geometry *g) {
    if (!d) return false;
    if (d->dtype != DCN4_F32 && d->dtype != DCN4_BF16 && d->dtype != DCN4_F16) return false;
    if (d->algo != DCN4_ALGO_AUTO && d->algo != DCN4_ALGO_GENERIC && d->algo != DCN4_ALGO_HALO &&
        d->algo != DCN4_ALGO_VECTOR)
        return false;
    if (d->math != DCN4_MATH_DEFAULT && d->math != DCN4_MATH_F32 && d->math != DCN4_MATH_MIXED16 &&
        d->math != DCN4_MATH_PACKED16 && d->math != DCN4_MATH_ACC16)
        return false;
    if (d->weights != DCN4_WEIGHTS_PLAIN && d->weights != DCN4_WEIGHTS_SOFTMAX) return false;
    if (d->msdcn_mode != DCN4_MSDCN_SCALE_OFFSET && d->msdcn_mode != DCN4_MSDCN_SCALE_DILATION)
        return false;
    int Ho = 0, Wo = 0;
    if (!out_hw(*d, &Ho, &Wo)) return false;
    const int K = d->kh * d->kw;
    const long long in_el = (long long)d->N * d->H * d->W * d->C;
    const long long out_el = (long long)d->N * Ho * Wo * d->C;
    const long long ow_el = (long long)d->N * Ho * Wo * d->G * K * 3;
    if (in_el > kMaxElems || out_el > kMaxElems || ow_el > kMaxElems) return false;
    if (!(d->offset_scale == d->offset_scale)) return false;  // NaN
    *g = Geometry{d->N, d->H, d->W, d->C, d->G, d->C / d->G, d->kh, d->kw, K,
                  d->stride_h, d->stride_w, d->pad_h, d->pad_w, d->dil_h, d->dil_w,
                  Ho, Wo, d->offset_scale, d->weights == DCN4_WEIGHTS_SOFTMAX ? 1 : 0,
                  d->msdcn_mode == DCN4_MSDCN_SCALE_DILATION ? 1 : 0};
    return true;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int ceil_to(int v, int m) { return (v + m - 1) / m * m; }

int log2_exact(int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return (1 << l) == v ? l : -1;
}

// Smallest power of two >= v.
int pow2_ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Chooses the halo kernel's tiling; false when the call does not fit it.
// The staged pixel (Gc groups x D channels) must be exactly 128 bytes, the
// stride at which random 16-byte gathers can be kept free of bank conflicts.
bool plan_halo(const Geometry &g, int eb, bool msdcn, bool rec_tma, HaloPlan *out) {
    if (128 % (g.D * eb) != 0) return false;
    const int Gc = 128 / (g.D * eb);
    if (g.G % Gc != 0) return false;
    const int U = g.D * eb / 16;
    const int smem_max = max_smem_optin();
    // record slots. Per-pixel bulk copies: room for the 16-byte superset copy
    // plus a word of read slack, stride 16 (mod 128) bytes. One TMA tile copy
    // per tile (rec_tma): the group slice starting at the 16-byte boundary
    // at or below it, rec_box elements per pixel.
    const int al = 16 / eb;
    const int rec_box = ceil_to(Gc * 27 + al - 1, al);
    const int slot = rec_tma ? rec_box * eb : ceil_to(Gc * 27 * eb + 16, 128) + 16;
    auto try_tile = [&](int TH, int TW, bool force_full, int stages, HaloPlan *p, int R) {
        if (stages == 2 && U > 4) return false;  // 16 warps need <= 128 registers
        TH = TH < g.Ho ? TH : g.Ho;
        TW = TW < pow2_ceil(g.Wo) ? TW : pow2_ceil(g.Wo);
        int HR = (TH - 1) * g.sh + (g.kh - 1) * g.dh + 2 * R + 2;
        int HC = (TW - 1) * g.sw + (g.kw - 1) * g.dw + 2 * R + 2;
        int full_h = force_full || HR >= g.H + 2;
        int full_w = force_full || HC >= g.W + 2;
        if (full_h) HR = g.H + 2;
        if (full_w) HC = g.W + 2;
        if (HR > 256 || HC > 256) return false;
        const long long halo = (long long)HR * HC * 128;
        HaloPlan q{TH, TW, Gc, log2_exact(TW), log2_exact(Gc), R, HR, HC, full_h, full_w,
                   (g.Ho + TH - 1) / TH, (g.Wo + TW - 1) / TW, g.G / Gc,
                   slot, (int)halo, stages, 0, rec_tma ? 1 : 0, rec_box};
        const long long total = (long long)stages *
                                    ((((halo + (long long)TH * TW * slot) + 127) / 128 * 128) +
                                     8 * (2 + 16));
        if ((long long)TH * TW * Gc > 1024) return false;
        if (total > smem_max) return false;
        q.smem_bytes = (int)total;
        *p = q;
        return true;
    };
    static const int cands[][2] = {{16, 8}, {8, 16}, {16, 16}, {8, 8}, {8, 4}, {4, 8},
                                   {4, 4}, {4, 2}, {2, 4}, {2, 2}, {2, 1}, {1, 2}, {1, 1}};
    // MSDCN offsets scale with s up to Smax: the whole image when it fits,
    // else the widest window (R <= 8) a two-stage 16 x 8 tile allows
    // (measured on the InternImage shape: R = 5 two-stage beats R = 8
    // one-stage and 8 x 8 tiles), else R = 8 on smaller tiles
    if (msdcn) {
        static const int big[][2] = {{32, 32}, {16, 32}, {32, 16}, {16, 16}, {8, 16}, {16, 8}, {8, 8}};
        for (auto &c : big)
            if (try_tile(c[0], c[1], true, 1, out, 8)) return true;
        for (int R = 8; R >= 5; --R)
            if (try_tile(16, 8, false, 2, out, R)) return true;
    }
    // DCNv4: R = 5 where the tile still fits (measured: 16x8 bf16 c2 120 ->
    // 110 us, fp32 194 -> 168 us, fewer samples take the global path),
    // else R = 4; the tile shape takes precedence over the radius
    const int Rs[2] = {msdcn ? 8 : 5, msdcn ? 8 : 4};
    for (int stages : {2, 1})
        for (auto &c : cands)
            for (int R : Rs)
                if (try_tile(c[0], c[1], false, stages, out, R)) return true;
    return false;
}

// Tiling and shared-memory layout of the backward halo kernel: one
// (pixel, group) pair per thread, or per four lanes when a group is 8 chunks
// (128 bytes: each lane owns 2); 256 or 512 threads; 128-byte staged pixels.
// The window reaches R = 4 pixels beyond the tile; for the multi-scale
// variant, whose scaled offsets reach far, the whole image (plus its zero
// border) is tried first. The sorted sample records (16 bytes each) and the
// owner list reuse the window and record slots, so they must fit there.
bool plan_bwd(const Geometry &g, int eb, bool rec_tma, bool msdcn, HaloPlan *out,
              BwdLayout *lay) {
    if (128 % (g.D * eb) != 0) return false;
    const int Gc = 128 / (g.D * eb);
    if (g.G % Gc != 0) return false;
    const int U = g.D * eb / 16;
    if (!(U == 4 || (U == 2 && eb == 2) || U == 8)) return false;
    const int lpp = U == 8 ? 4 : 1;
    const int R = 4;
    const int smem_max = max_smem_optin() - 1024;  // static shared memory of the kernel
    // record slots as in plan_halo: per-pixel bulk copies, or one TMA tile copy
    const int al = 16 / eb;
    const int rec_box = ceil_to(Gc * 27 + al - 1, al);
    const int slot = rec_tma ? rec_box * eb : ceil_to(Gc * 27 * eb + 16, 128) + 16;
    const int per_sm = max_smem_per_sm();
    // tile (TH, TW), whole-image window or not; `first` demands a 256-pair
    // tile that runs two CTAs per SM (the phases of one CTA then overlap the
    // other's)
    auto try_plan = [&](int TH, int TW, bool force_full, bool first) -> bool {
        TH = TH < g.Ho ? TH : g.Ho;
        TW = TW < pow2_ceil(g.Wo) ? TW : pow2_ceil(g.Wo);
        const int pairs = TH * TW * Gc;
        if (pairs * lpp > 512) return false;
        int HR = (TH - 1) * g.sh + (g.kh - 1) * g.dh + 2 * R + 2;
        int HC = (TW - 1) * g.sw + (g.kw - 1) * g.dw + 2 * R + 2;
        const int full_h = force_full || HR >= g.H + 2, full_w = force_full || HC >= g.W + 2;
        if (full_h) HR = g.H + 2;
        if (full_w) HC = g.W + 2;
        if (HR > 256 || HC > 256 || TH > 256 || TW > 256) return false;
        const int halo = HR * HC * 128;
        const int max_samples = pairs * 9;
        const int ncells = (HR - 1) * (HC - 1) * Gc;
        const int nown = HR * HC * Gc;
        // sorted samples (16 bytes each), then the owner list and the owners'
        // ranks (2 bytes each per staged (pixel, group)) and their counts
        // (1 byte each) reuse the window and record slots
        const int olist_off = ceil_to(16 * max_samples, 16);
        if (olist_off + 5 * nown > halo + TH * TW * slot || ncells > 65535 || nown > 65535)
            return false;
        BwdLayout L;
        // window and record slots first: both are free after phase A
        L.slots_off = halo;
        L.go_off = ceil_to(L.slots_off + TH * TW * slot, 128);  // TMA destination
        L.gows_off = L.go_off + TH * TW * 128;
        L.counts_off = ceil_to(L.gows_off + TH * TW * Gc * 27 * eb, 16);
        L.bar_off = ceil_to(L.counts_off + (ncells + 1) * 4, 16);
        L.ncells = ncells;
        L.max_samples = max_samples;
        L.olist_off = olist_off;
        L.hc_magic = (unsigned)(((1ull << 32) + HC - 1) / HC);
        L.smem_bytes = L.bar_off + 16;
        if (L.smem_bytes > smem_max) return false;
        const bool two = pairs * lpp <= 256 && 2 * (L.smem_bytes + 1024 + 1024) <= per_sm;
        if (first && !(two && pairs * lpp == 256)) return false;
        L.threads = two ? 256 : 512;
        L.lpp = lpp;
        *out = HaloPlan{TH, TW, Gc, log2_exact(TW), log2_exact(Gc), R, HR, HC, full_h, full_w,
                        (g.Ho + TH - 1) / TH, (g.Wo + TW - 1) / TW, g.G / Gc, slot, halo, 1,
                        L.smem_bytes, rec_tma ? 1 : 0, rec_box};
        *lay = L;
        return true;
    };
    static const int cands[][2] = {{16, 8}, {8, 16}, {8, 8}, {8, 4}, {4, 8},
                                   {4, 4}, {4, 2}, {2, 4}, {2, 2}, {2, 1}, {1, 2}, {1, 1}};
    if (msdcn && lpp > 1) {  // wide groups: the whole image when it fits
        for (auto &c : cands)
            if (try_plan(c[0], c[1], true, false)) return true;
    }
    if (try_plan(8, 8, false, true)) return true;
    for (auto &c : cands)
        if (try_plan(c[0], c[1], false, false)) return true;
    return false;
}

// Tiling and shared-memory carve-up of the fused producer + forward kernel:
// 16-bit data, 3x3 taps, 128-byte staged pixels of Gc groups with 2 or 4
// chunks each (so C is a multiple of 64: whole MMA K steps and whole blocks
// of 8 depthwise chunks), C <= 256 (one TMA box row), the offset grid equal
// to the input grid. One stage: the input window (reach R,
// 5 where the tile fits, else 4 or 3), the record slots, x's neighbourhood
// of the tile, A (128 rows), the slice's lin_w rows, taps and biases; a tile
// of at most 128 pixels (the MMA's M).
bool plan_fused(const Geometry &g, int eb, HaloPlan *out, FusedLayout *lay) {
    if (eb != 2 || g.kh != 3 || g.kw != 3) return false;
    if (g.Ho != g.H || g.Wo != g.W) return false;
    if ((g.D * eb) % 16 != 0) return false;
    const int U = g.D * eb / 16;
    if (U != 2 && U != 4) return false;
    if (g.C % 64 != 0 || g.C > 256) return false;
    const int Gc = 128 / (g.D * eb);
    if (g.G % Gc != 0) return false;
    const int JS = Gc * 27, NP = ceil_to(JS, 16);
    const int slot = NP * eb + 16;  // an odd multiple of 16 bytes
    const int smem_max = max_smem_optin();
    auto try_tile = [&](int TH, int TW, int R) -> bool {
        TH = TH < g.Ho ? TH : g.Ho;
        TW = TW < pow2_ceil(g.Wo) ? TW : pow2_ceil(g.Wo);
        if (TH * TW > 128) return false;
        int HR = (TH - 1) * g.sh + (g.kh - 1) * g.dh + 2 * R + 2;
        int HC = (TW - 1) * g.sw + (g.kw - 1) * g.dw + 2 * R + 2;
        const int full_h = HR >= g.H + 2, full_w = HC >= g.W + 2;
        if (full_h) HR = g.H + 2;
        if (full_w) HC = g.W + 2;
        if (HR > 256 || HC > 256) return false;
        const int halo = HR * HC * 128;
        FusedLayout L;
        L.win_off = 0;
        L.slots_off = ceil_to(halo, 128);
        L.x_off = ceil_to(L.slots_off + TH * TW * slot, 128);
        L.x_bytes = (TH + 2) * (TW + 2) * g.C * eb;
        L.a_off = ceil_to(L.x_off + L.x_bytes, 1024);
        L.b_off = L.a_off + 128 * g.C * eb;
        L.dwt_off = L.b_off + NP * g.C * eb;
        L.dwb_off = ceil_to(L.dwt_off + 9 * g.C * eb, 16);
        L.linb_off = L.dwb_off + g.C * 4;
        L.bar_off = ceil_to(L.linb_off + NP * 4, 16);
        L.bytes = L.bar_off + 32;
        L.JS = JS;
        L.NP = NP;
        L.tmem_cols = 32;
        while (L.tmem_cols < NP) L.tmem_cols <<= 1;
        if (L.bytes > smem_max) return false;
        *out = HaloPlan{TH, TW, Gc, log2_exact(TW), log2_exact(Gc), R, HR, HC, full_h, full_w,
                        (g.Ho + TH - 1) / TH, (g.Wo + TW - 1) / TW, g.G / Gc, slot, halo, 1,
                        L.bytes, 2, 0};
        *lay = L;
        return true;
    };
    static const int cands[][2] = {{16, 8}, {8, 16}, {8, 8}, {8, 4}, {4, 8}, {4, 4},
                                   {4, 2},  {2, 4},  {2, 2}, {2, 1}, {1, 2}, {1, 1}};
    for (auto &c : cands)
        for (int R : {5, 4, 3})
            if (try_tile(c[0], c[1], R)) return true;
    return false;
}

// Tiling and shared-memory carve-up of the 2-D tiled tensor-core producer:
// 16-bit data, C a multiple of 64 (whole blocks of 8 depthwise chunks) and at
// most 256 (one TMA box row), J <= 256 outputs in whole 16-byte rows (the TMA
// store's inner box). Tiles of at most 128 pixels (the MMA's M), 16 x 8 first.
bool plan_producer_2d(int H, int W, int C, int J, int NP, ProducerTc2dLayout *out) {
    if (C % 64 != 0 || C > 256 || J > 256 || (J * 2) % 16 != 0) return false;
    const int smem_max = max_smem_optin();
    static const int cands[][2] = {{16, 8}, {8, 16}, {8, 8}, {8, 4}, {4, 8}, {4, 4},
                                   {4, 2},  {2, 4},  {2, 2}, {2, 1}, {1, 2}, {1, 1}};
    for (auto &c : cands) {
        const int TH = c[0] < H ? c[0] : H;
        const int TW = c[1] < pow2_ceil(W) ? c[1] : pow2_ceil(W);
        if (TH * TW > 128) continue;
        ProducerTc2dLayout L;
        L.TH = TH;
        L.TW = TW;
        L.lgTW = log2_exact(TW);
        L.tiles_h = (H + TH - 1) / TH;
        L.tiles_w = (W + TW - 1) / TW;
        L.x_off = 0;
        L.x_bytes = (TH + 2) * (TW + 2) * C * 2;
        L.a_off = ceil_to(L.x_off + L.x_bytes, 1024);
        L.b_off = L.a_off + 128 * C * 2;
        L.o_off = ceil_to(L.b_off + NP * C * 2, 1024);
        L.dwt_off = ceil_to(L.o_off + TH * TW * J * 2, 16);
        L.dwb_off = ceil_to(L.dwt_off + 9 * C * 2, 16);
        L.linb_off = L.dwb_off + C * 4;
        L.bar_off = ceil_to(L.linb_off + NP * 4, 16);
        L.bytes = L.bar_off + 32;
        L.tmem_cols = 32;
        while (L.tmem_cols < NP) L.tmem_cols <<= 1;
        if (L.bytes > smem_max) continue;
        *out = L;
        return true;
    }
    return false;
}

// Where the fused kernel splits a tile's groups over several slices, each
// slice's CTA repeats the depthwise pass and runs the gathers with one CTA
// per SM after it; the two-kernel chain is then the faster one when the 2-D
// tensor-core producer takes the shape in one pass (J <= 256 outputs,
// lin_w resident; InternImage stage, N64 56x56 C128 G8 bf16: 166-174 us
// against 225 us), or when there are 4 slices or more, whose producer (the
// fused kernel's producer steps alone) and forward run apart faster (C256
// G16: 285 against 369 us; C256 G8: 684 against 829 us). With 2 or 3
// slices and that producer the two are within a few percent (C128 G4: 266
// against 248 us; C192 G12: 477 against 471 us) and one slice favours the
// fused kernel (C64 G4: 111 against 141 us).
bool chain_preferred(const Geometry &g, int eb, const HaloPlan &fused_plan) {
    if (fused_plan.slices < 2 || eb != 2) return false;
    if (fused_plan.slices >= 4) return true;
    const int J = g.G * g.K * 3, NP = (J + 15) / 16 * 16;
    if (g.C % 16 != 0 || NP > 256 || (J * eb) % 16 != 0) return false;
    ProducerTcLayout lay = ProducerTcLayout::make(g.C, J, NP, g.W, 2);
    if (lay.bytes > max_smem_optin()) lay = ProducerTcLayout::make(g.C, J, NP, g.W, 1);
    if (lay.bytes > max_smem_optin()) return false;
    ProducerTc2dLayout l2;
    return plan_producer_2d(g.H, g.W, g.C, J, NP, &l2);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// TMA descriptor of a channel-last [N][rows][cols][C] tensor with a box of
// (box_c channels, box_w columns, box_h rows, 1 image); zero fill out of bounds.
bool encode_map(Dtype dt, const void *base, int N, int rows, int cols, int C, int box_c,
                int box_w, int box_h, CUtensorMap *map) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int eb = elem_bytes(dt);
    const CUtensorMapDataType t = dt == Dtype::F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dt == Dtype::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)N};
    cuuint64_t strides[3] = {(cuuint64_t)C * eb, (cuuint64_t)cols * C * eb,
                             (cuuint64_t)rows * cols * C * eb};
    cuuint32_t box[4] = {(cuuint32_t)box_c, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, t, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// TMA descriptor of the input viewed as [N][H][W][C] with a box of
// (Gc*D channels, HC columns, HR rows, 1 image); zero fill out of bounds.
bool encode_input_map(const Geometry &g, Dtype dt, const void *in, const HaloPlan &p,
                      CUtensorMap *map) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int eb = elem_bytes(dt);
    const CUtensorMapDataType t = dt == Dtype::F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dt == Dtype::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[4] = {(cuuint64_t)g.C, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.N};
    cuuint64_t strides[3] = {(cuuint64_t)g.C * eb, (cuuint64_t)g.W * g.C * eb,
                             (cuuint64_t)g.H * g.W * g.C * eb};
    cuuint32_t box[4] = {(cuuint32_t)(p.Gc * g.D), (cuuint32_t)p.HC, (cuuint32_t)p.HR, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, t, 4, const_cast<void *>(in), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Whether the halo kernel can run this call; fills plan and tensor maps.
// The records arrive by TMA (map_ow) when a pixel's G*27 values span a
// multiple of 16 bytes (the TMA stride rule), else by per-pixel bulk copies.
bool halo_ok(const Geometry &g, Dtype dt, bool msdcn, const void *in, const void *ow,
             const void *out, HaloPlan *plan, CUtensorMap *map, CUtensorMap *map_ow) {
    const int eb = elem_bytes(dt);
    if (g.kh != 3 || g.kw != 3) return false;
    if ((g.D * eb) % 16 != 0) return false;
    const int U = g.D * eb / 16;
    if (U != 2 && U != 4 && U != 8) return false;
    if (eb == 4 && U == 2) return false;
    if (!aligned16(in) || !aligned16(ow) || !aligned16(out)) return false;
    const bool rec_tma = (g.G * 27 * eb) % 16 == 0;
    if (rec_tma && plan_halo(g, eb, msdcn, true, plan) &&
        encode_map(dt, ow, g.N, g.Ho, g.Wo, g.G * 27, plan->rec_box, plan->TW, plan->TH, map_ow) &&
        encode_input_map(g, dt, in, *plan, map))
        return true;
    if (!plan_halo(g, eb, msdcn, false, plan)) return false;
    return encode_input_map(g, dt, in, *plan, map);
}

dcn4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DCN4_OK : DCN4_ERR_CUDA; }

// Whether the 16-bit kernels round the bilinear weights to the data type.
// 16-bit weights (mixed-precision fma) in the backward's gather of grad_input
bool use_mixed(const dcn4_desc *d) {
    if (d->dtype == DCN4_F32) return false;
    return d->math == DCN4_MATH_MIXED16 || d->math == DCN4_MATH_DEFAULT ||
           d->math == DCN4_MATH_PACKED16 || d->math == DCN4_MATH_ACC16;
}

// forward multiply variant: 0 fp32 weights, 1 mixed-precision fma, 2 packed
int forward_math(const dcn4_desc *d) {
    if (d->dtype == DCN4_F32 || d->math == DCN4_MATH_F32) return 0;
    return d->math == DCN4_MATH_PACKED16 ? 2 : 1;
}

dcn4_status run_forward(const dcn4_desc *desc, const void *input, const void *ow, void *output,
                        void *stream, const MsdcnParams *ms, void *ws = nullptr,
                        size_t ws_bytes = 0) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!input || !ow || !output) return DCN4_ERR_INVALID_ARG;
    if (ms && !ms->raw) return DCN4_ERR_INVALID_ARG;
    FwdLaunch L;
    memset(&L, 0, sizeof(L));
    L.geo = g;
    L.dtype = static_cast<Dtype>(desc->dtype);
    L.msdcn = ms != nullptr;
    L.in = input;
    L.ow = ow;
    L.out = output;
    L.ms = ms;
    L.mathv = forward_math(desc);
    L.stream = static_cast<cudaStream_t>(stream);
    L.ow_bytes = (unsigned long long)g.N * g.Ho * g.Wo * g.G * g.K * 3 * elem_bytes(L.dtype);
    if (ws != nullptr && aligned16(ws)) {
        L.ws = ws;
        L.ws_bytes = ws_bytes;
    }
    CUtensorMap map, map_ow;
    memset(&map, 0, sizeof(map));
    memset(&map_ow, 0, sizeof(map_ow));
    if (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_HALO) {
        L.halo = halo_ok(g, L.dtype, L.msdcn, input, ow, output, &L.plan, &map, &map_ow);
        if (!L.halo && desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    }
    if (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_VECTOR) {
        // vectorised global-memory kernel: whole 16-byte vectors per group,
        // 16-byte aligned input and output
        const int eb = elem_bytes(L.dtype);
        L.vec = !L.halo && (g.D * eb) % 16 == 0 && aligned16(input) && aligned16(output);
        if (!L.vec && desc->algo == DCN4_ALGO_VECTOR) return DCN4_ERR_UNSUPPORTED;
    }
    L.tmap = &map;
    L.tmap_ow = &map_ow;
    return cuda_status(launch_forward(L));
}

}  // namespace

extern "C" {

dcn4_status dcn4_out_shape(const dcn4_desc *desc, int *Ho, int *Wo) {
    Geometry g;
    if (!make_geometry(desc, &g) || !Ho || !Wo) return DCN4_ERR_INVALID_ARG;
    *Ho = g.Ho;
    *Wo = g.Wo;
    return DCN4_OK;
}

dcn4_status dcn4_forward(const dcn4_desc *desc, const void *input, const void *offset_weight,
                         void *output, void *stream) {
    return run_forward(desc, input, offset_weight, output, stream, nullptr);
}

dcn4_status dcn4_forward_workspace_size(const dcn4_desc *desc, size_t *bytes) {
    Geometry g;
    if (!make_geometry(desc, &g) || !bytes) return DCN4_ERR_INVALID_ARG;
    const int eb = elem_bytes(static_cast<Dtype>(desc->dtype));
    // the staged kernel with one lane per (pixel, group): 3x3 taps, groups of
    // 2 (16-bit) or 4 16-byte chunks
    const int U = (g.D * eb) % 16 == 0 ? g.D * eb / 16 : 0;
    const bool staged = g.kh == 3 && g.kw == 3 && (U == 4 || (U == 2 && eb == 2)) &&
                        (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_HALO);
    *bytes = staged ? forward_escape_bytes((long long)g.N * g.Ho * g.Wo * g.G, g.D, eb,
                                           sm_count() * 8)
                    : 0;
    return DCN4_OK;
}

dcn4_status dcn4_forward_ws(const dcn4_desc *desc, const void *input, const void *offset_weight,
                            void *output, void *workspace, size_t workspace_bytes, void *stream) {
    return run_forward(desc, input, offset_weight, output, stream, nullptr, workspace,
                       workspace_bytes);
}

dcn4_status dcn4_offset_producer(const dcn4_desc *desc, const void *x, const void *dw_weight,
                                 const void *dw_bias, const void *lin_weight,
                                 const void *lin_bias, void *offset_weight, void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!x || !dw_weight || !dw_bias || !lin_weight || !lin_bias || !offset_weight)
        return DCN4_ERR_INVALID_ARG;
    if (g.Ho != g.H || g.Wo != g.W) return DCN4_ERR_UNSUPPORTED;
    ProducerLaunch L;
    memset(&L, 0, sizeof(L));
    L.dtype = static_cast<Dtype>(desc->dtype);
    L.pg.N = g.N;
    L.pg.H = g.H;
    L.pg.W = g.W;
    L.pg.C = g.C;
    L.pg.J = g.G * g.K * 3;
    L.pg.NP = (L.pg.J + 15) / 16 * 16;
    L.pg.npix = (long long)g.N * g.H * g.W;
    const long long ntiles = (L.pg.npix + 127) / 128;
    if (L.pg.npix + 128 > std::numeric_limits<int>::max()) return DCN4_ERR_UNSUPPORTED;
    L.pg.ntiles = (int)ntiles;
    L.x = x;
    L.dw_w = dw_weight;
    L.dw_b = dw_bias;
    L.lin_w = lin_weight;
    L.lin_b = lin_bias;
    L.out = offset_weight;
    L.stream = static_cast<cudaStream_t>(stream);
    const int eb = elem_bytes(L.dtype);
    // tensor-core kernel: 16-bit data, K = C in steps of 16, N = J padded to
    // 16 <= 256, whole 16-byte output rows, lin_w resident in shared memory
    ProducerTcLayout lay = ProducerTcLayout::make(g.C, L.pg.J, L.pg.NP, g.W, 2);
    if (lay.bytes > max_smem_optin()) lay = ProducerTcLayout::make(g.C, L.pg.J, L.pg.NP, g.W, 1);
    L.tc = desc->algo != DCN4_ALGO_GENERIC && eb == 2 && g.C % 16 == 0 && L.pg.NP <= 256 &&
           (L.pg.J * eb) % 16 == 0 && aligned16(x) && aligned16(lin_weight) &&
           aligned16(offset_weight) && lay.bytes <= max_smem_optin();
    L.lay = lay;
    if (!L.tc && desc->algo != DCN4_ALGO_GENERIC && eb == 2) {
        // the fused kernel's producer steps alone: a slice of the groups'
        // outputs per CTA on the tensor cores, records written out
        FusedLaunch F;
        memset(&F, 0, sizeof(F));
        CUtensorMap map_in, map_xs;
        memset(&map_in, 0, sizeof(map_in));
        memset(&map_xs, 0, sizeof(map_xs));
        if (plan_fused(g, eb, &F.plan, &F.lay) && aligned16(x) && aligned16(lin_weight) &&
            (reinterpret_cast<uintptr_t>(offset_weight) & 3) == 0 &&
            encode_input_map(g, L.dtype, x, F.plan, &map_in) &&
            encode_map(L.dtype, x, g.N, g.H, g.W, g.C, g.C, F.plan.TW + 2, F.plan.TH + 2,
                       &map_xs)) {
            F.geo = g;
            F.dtype = L.dtype;
            F.in = x;  // no window is loaded; the map only fills the argument
            F.x = x;
            F.dw_w = dw_weight;
            F.dw_b = dw_bias;
            F.lin_w = lin_weight;
            F.lin_b = lin_bias;
            F.out = nullptr;
            F.rec_out = offset_weight;
            F.records_only = true;
            F.mathv = 1;
            F.tmap_in = &map_in;
            F.tmap_x = &map_xs;
            F.stream = L.stream;
            return cuda_status(launch_fused(F));
        }
    }
    if (!L.tc && desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    // the 2-D tiled kernel where it applies (x by TMA tile, sliding-window
    // depthwise, one TMA store per tile)
    CUtensorMap map_x, map_out;
    memset(&map_x, 0, sizeof(map_x));
    memset(&map_out, 0, sizeof(map_out));
    L.tc2d = L.tc && plan_producer_2d(g.H, g.W, g.C, L.pg.J, L.pg.NP, &L.lay2) &&
             encode_map(L.dtype, x, g.N, g.H, g.W, g.C, g.C, L.lay2.TW + 2, L.lay2.TH + 2,
                        &map_x) &&
             encode_map(L.dtype, offset_weight, g.N, g.H, g.W, L.pg.J, L.pg.J, L.lay2.TW,
                        L.lay2.TH, &map_out) &&
             (long long)g.N * L.lay2.tiles_h * L.lay2.tiles_w <= 0x7fffffffLL;
    L.tmap_x = &map_x;
    L.tmap_out = &map_out;
    if (!L.tc && (L.pg.npix + kProducerPixels - 1) / kProducerPixels > 0x7fffffffLL)
        return DCN4_ERR_UNSUPPORTED;
    return cuda_status(launch_producer(L));
}

dcn4_status dcn4_fused_forward_workspace_size(const dcn4_desc *desc, size_t *bytes) {
    Geometry g;
    if (!make_geometry(desc, &g) || !bytes) return DCN4_ERR_INVALID_ARG;
    HaloPlan plan;
    FusedLayout lay;
    const int eb = elem_bytes(static_cast<Dtype>(desc->dtype));
    const bool fused = (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_HALO) &&
                       plan_fused(g, eb, &plan, &lay) &&
                       !(desc->algo == DCN4_ALGO_AUTO && chain_preferred(g, eb, plan));
    if (fused) {
        *bytes = 0;
        return DCN4_OK;
    }
    // the chain: the records, then scratch for the forward's escapes
    size_t esc = 0;
    dcn4_forward_workspace_size(desc, &esc);
    *bytes = ((size_t)g.N * g.Ho * g.Wo * g.G * g.K * 3 * (size_t)eb + 15) / 16 * 16 + esc;
    return DCN4_OK;
}

dcn4_status dcn4_fused_forward(const dcn4_desc *desc, const void *input, const void *x,
                               const void *dw_weight, const void *dw_bias,
                               const void *lin_weight, const void *lin_bias, void *output,
                               void *offset_weight_out, void *workspace, size_t workspace_bytes,
                               void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!input || !x || !dw_weight || !dw_bias || !lin_weight || !lin_bias || !output)
        return DCN4_ERR_INVALID_ARG;
    if (g.Ho != g.H || g.Wo != g.W) return DCN4_ERR_UNSUPPORTED;
    const Dtype dt = static_cast<Dtype>(desc->dtype);
    const int eb = elem_bytes(dt);
    if (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_HALO) {
        FusedLaunch L;
        memset(&L, 0, sizeof(L));
        CUtensorMap map_in, map_x;
        memset(&map_in, 0, sizeof(map_in));
        memset(&map_x, 0, sizeof(map_x));
        const bool fused =
            plan_fused(g, eb, &L.plan, &L.lay) && aligned16(input) && aligned16(x) &&
            aligned16(lin_weight) && aligned16(output) &&
            (reinterpret_cast<uintptr_t>(offset_weight_out) & 3) == 0 &&
            encode_input_map(g, dt, input, L.plan, &map_in) &&
            encode_map(dt, x, g.N, g.H, g.W, g.C, g.C, L.plan.TW + 2, L.plan.TH + 2, &map_x);
        // AUTO takes the chain where it is faster, when there is room for
        // the records (aligned for the producer's TMA store)
        void *rec = offset_weight_out;
        const size_t rec_bytes = (size_t)g.N * g.Ho * g.Wo * g.G * g.K * 3 * (size_t)eb;
        if (!rec && workspace && workspace_bytes >= rec_bytes) rec = workspace;
        const bool to_chain = fused && desc->algo == DCN4_ALGO_AUTO &&
                              chain_preferred(g, eb, L.plan) && rec != nullptr && aligned16(rec) &&
                              aligned16(lin_weight);
        if (fused && !to_chain) {
            L.geo = g;
            L.dtype = dt;
            L.in = input;
            L.x = x;
            L.dw_w = dw_weight;
            L.dw_b = dw_bias;
            L.lin_w = lin_weight;
            L.lin_b = lin_bias;
            L.out = output;
            L.rec_out = offset_weight_out;
            L.mathv = forward_math(desc);
            L.tmap_in = &map_in;
            L.tmap_x = &map_x;
            L.stream = static_cast<cudaStream_t>(stream);
            return cuda_status(launch_fused(L));
        }
        if (!fused && desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    }
    // the two-kernel chain, through offset_weight_out when given, else
    // through the caller's scratch
    void *records = offset_weight_out;
    void *esc = workspace;  // what the records leave of the scratch: the forward's escapes
    size_t esc_bytes = workspace ? workspace_bytes : 0;
    if (!records) {
        const size_t need = (size_t)g.N * g.Ho * g.Wo * g.G * g.K * 3 * (size_t)eb;
        if (!workspace || workspace_bytes < need) return DCN4_ERR_WORKSPACE;
        records = workspace;
        const size_t used = (need + 15) / 16 * 16;
        esc = workspace_bytes > used ? static_cast<unsigned char *>(workspace) + used : nullptr;
        esc_bytes = workspace_bytes > used ? workspace_bytes - used : 0;
    }
    dcn4_desc d = *desc;
    d.algo = desc->algo == DCN4_ALGO_GENERIC ? DCN4_ALGO_GENERIC : DCN4_ALGO_AUTO;
    const dcn4_status st =
        dcn4_offset_producer(&d, x, dw_weight, dw_bias, lin_weight, lin_bias, records, stream);
    if (st != DCN4_OK) return st;
    d.algo = desc->algo;
    return dcn4_forward_ws(&d, input, records, output, esc, esc_bytes, stream);
}

dcn4_status dcn4_backward_workspace_size(const dcn4_desc *desc, size_t *bytes) {
    Geometry g;
    if (!make_geometry(desc, &g) || !bytes) return DCN4_ERR_INVALID_ARG;
    *bytes = desc->dtype == DCN4_F32 ? 0 : (size_t)g.N * g.H * g.W * g.C * sizeof(float);
    return DCN4_OK;
}

}  // extern "C"

namespace {

// Shared by dcn4_backward and msdcn_backward (ms != nullptr: the FlowDCN
// multi-scale variant, graw receives the gradient of scale_raw).
dcn4_status run_backward(const dcn4_desc *desc, const void *input, const void *offset_weight,
                         const void *grad_out, void *grad_input, void *grad_offset_weight,
                         void *workspace, size_t workspace_bytes, void *stream,
                         const MsdcnParams *ms, void *graw) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!input || !offset_weight || !grad_out || !grad_input || !grad_offset_weight)
        return DCN4_ERR_INVALID_ARG;
    if (ms && !graw) return DCN4_ERR_INVALID_ARG;
    size_t need = 0;
    dcn4_backward_workspace_size(desc, &need);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DCN4_ERR_WORKSPACE;
    BwdLaunch L;
    memset(&L, 0, sizeof(L));
    L.geo = g;
    L.dtype = static_cast<Dtype>(desc->dtype);
    L.in = input;
    L.ow = offset_weight;
    L.gout = grad_out;
    L.gin = grad_input;
    L.gow = grad_offset_weight;
    L.acc = need > 0 ? static_cast<float *>(workspace) : static_cast<float *>(grad_input);
    L.mixed = use_mixed(desc);
    L.acc16 = desc->math == DCN4_MATH_ACC16;
    L.stream = static_cast<cudaStream_t>(stream);
    L.msdcn = ms != nullptr;
    L.ms = ms;
    L.graw = graw;
    const int eb = elem_bytes(L.dtype);
    L.ow_bytes = (unsigned long long)g.N * g.Ho * g.Wo * g.G * g.K * 3 * eb;
    CUtensorMap map_in, map_go, map_ow;
    memset(&map_in, 0, sizeof(map_in));
    memset(&map_go, 0, sizeof(map_go));
    memset(&map_ow, 0, sizeof(map_ow));
    if (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_HALO) {
        const bool base = g.kh == 3 && g.kw == 3 && aligned16(input) &&
                          aligned16(offset_weight) && aligned16(grad_out) && aligned16(L.acc);
        auto maps = [&]() {
            return encode_input_map(g, L.dtype, input, L.plan, &map_in) &&
                   encode_map(L.dtype, grad_out, g.N, g.Ho, g.Wo, g.C, L.plan.Gc * g.D,
                              L.plan.TW, L.plan.TH, &map_go);
        };
        // records by one TMA tile copy when a pixel's G*27 values span a
        // multiple of 16 bytes, else by per-pixel bulk copies
        L.halo = base && (g.G * 27 * eb) % 16 == 0 && plan_bwd(g, eb, true, L.msdcn, &L.plan, &L.layout) &&
                 maps() &&
                 encode_map(L.dtype, offset_weight, g.N, g.Ho, g.Wo, g.G * 27, L.plan.rec_box,
                            L.plan.TW, L.plan.TH, &map_ow);
        if (!L.halo)
            L.halo = base && plan_bwd(g, eb, false, L.msdcn, &L.plan, &L.layout) && maps();
        if (!L.halo && desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    }
    // vectorised global-memory kernel: whole 16-byte vectors per group, a
    // power-of-two count of them (<= 16), 16-byte aligned tensors
    const int vb = g.D * eb;
    L.vec = !L.halo && (desc->algo == DCN4_ALGO_AUTO || desc->algo == DCN4_ALGO_VECTOR) &&
            vb % 16 == 0 && vb <= 256 && ((vb / 16) & (vb / 16 - 1)) == 0 && aligned16(input) &&
            aligned16(grad_out) && aligned16(L.acc);
    if (!L.vec && desc->algo == DCN4_ALGO_VECTOR) return DCN4_ERR_UNSUPPORTED;
    L.tmap_in = &map_in;
    L.tmap_go = &map_go;
    L.tmap_ow = &map_ow;
    return cuda_status(launch_backward(L));
}

}  // namespace

extern "C" {

dcn4_status dcn4_backward(const dcn4_desc *desc, const void *input, const void *offset_weight,
                          const void *grad_out, void *grad_input, void *grad_offset_weight,
                          void *workspace, size_t workspace_bytes, void *stream) {
    return run_backward(desc, input, offset_weight, grad_out, grad_input, grad_offset_weight,
                        workspace, workspace_bytes, stream, nullptr, nullptr);
}

dcn4_status msdcn_backward(const dcn4_desc *desc, const void *input, const void *dir_weight,
                           const void *scale_raw, const float *s0_host, float smax,
                           const void *grad_out, void *grad_input, void *grad_dir_weight,
                           void *grad_scale_raw, void *workspace, size_t workspace_bytes,
                           void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!s0_host || !scale_raw || !grad_scale_raw) return DCN4_ERR_INVALID_ARG;
    if (g.softmax) return DCN4_ERR_UNSUPPORTED;
    static thread_local MsdcnParams ms;
    ms.raw = scale_raw;
    ms.smax = smax;
    for (int i = 0; i < g.G; ++i) ms.s0[i] = s0_host[i];
    return run_backward(desc, input, dir_weight, grad_out, grad_input, grad_dir_weight,
                        workspace, workspace_bytes, stream, &ms, grad_scale_raw);
}

dcn4_status msdcn_forward(const dcn4_desc *desc, const void *input, const void *dir_weight,
                          const void *scale_raw, const float *s0_host, float smax, void *output,
                          void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!s0_host || !scale_raw) return DCN4_ERR_INVALID_ARG;
    if (g.softmax) return DCN4_ERR_UNSUPPORTED;
    static thread_local MsdcnParams ms;
    ms.raw = scale_raw;
    ms.smax = smax;
    for (int i = 0; i < g.G; ++i) ms.s0[i] = s0_host[i];
    return run_forward(desc, input, dir_weight, output, stream, &ms);
}

dcn4_status msdcn_forward_ws(const dcn4_desc *desc, const void *input, const void *dir_weight,
                             const void *scale_raw, const float *s0_host, float smax,
                             void *output, void *workspace, size_t workspace_bytes,
                             void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!s0_host || !scale_raw) return DCN4_ERR_INVALID_ARG;
    if (g.softmax) return DCN4_ERR_UNSUPPORTED;
    static thread_local MsdcnParams ms;
    ms.raw = scale_raw;
    ms.smax = smax;
    for (int i = 0; i < g.G; ++i) ms.s0[i] = s0_host[i];
    return run_forward(desc, input, dir_weight, output, stream, &ms, workspace, workspace_bytes);
}

const char *dcn4_status_string(dcn4_status s) {
    switch (s) {
        case DCN4_OK: return "DCN4_OK";
        case DCN4_ERR_INVALID_ARG: return "DCN4_ERR_INVALID_ARG";
        case DCN4_ERR_UNSUPPORTED: return "DCN4_ERR_UNSUPPORTED";
        case DCN4_ERR_WORKSPACE: return "DCN4_ERR_WORKSPACE";
        case DCN4_ERR_CUDA: return "DCN4_ERR_CUDA";
        case DCN4_ERR_TIMEOUT: return "DCN4_ERR_TIMEOUT";
        case DCN4_ERR_INTERNAL: return "DCN4_ERR_INTERNAL";
    }
    return "DCN4_UNKNOWN_STATUS";
}

dcn4_status dcn4_selftest_bounded_wait(unsigned int timeout_us, void *stream) {
    if (timeout_us < 1) timeout_us = 1;
    if (timeout_us > 2000000u) timeout_us = 2000000u;
    return cuda_status(
        launch_selftest_wait(1000ull * timeout_us, static_cast<cudaStream_t>(stream)));
}

dcn4_status dcn4_last_device_error(unsigned int *code) {
    if (!code) return DCN4_ERR_INVALID_ARG;
    unsigned bits = 0;
    if (read_clear_device_error(&bits) != cudaSuccess) return DCN4_ERR_CUDA;
    *code = bits;
    if (bits & kErrTimeout) return DCN4_ERR_TIMEOUT;
    if (bits & kErrInternal) return DCN4_ERR_INTERNAL;
    return DCN4_OK;
}

dcn4_status dcn4_kernel_launches(unsigned long long *count) {
    if (!count) return DCN4_ERR_INVALID_ARG;
    *count = launches_issued();
    return DCN4_OK;
}

}  // extern "C"
