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
    if (d->algo != DCN4_ALGO_AUTO && d->algo != DCN4_ALGO_GENERIC && d->algo != DCN4_ALGO_HALO)
        return false;
    if (d->math != DCN4_MATH_F32 && d->math != DCN4_MATH_MIXED16) return false;
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
                  Ho, Wo, d->offset_scale};
    return true;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int ceil_to(int v, int m) { return (v + m - 1) / m * m; }

// Chooses the halo kernel's tiling; false when no tiling fits shared memory.
bool plan_halo(const Geometry &g, int eb, bool msdcn, HaloPlan *out) {
    const int U = g.D * eb / 16;
    int Gc = 0;
    for (int d = 1; d <= g.G; ++d)
        if (g.G % d == 0 && (d * U) % 8 == 0 && d * g.D <= 256) { Gc = d; break; }
    if (Gc == 0) Gc = 1;
    if (Gc * g.D > 256) return false;
    const int R = msdcn ? 8 : 4;
    const int smem_max = max_smem_optin();
    const int budget_two = 110 * 1024;  // two CTAs per SM
    // record slots: room for the 16-byte superset copy plus a word of read
    // slack, and a stride of 16 (mod 128) bytes so that the records of
    // consecutive pixels start in different bank quads
    const int slot = ceil_to(Gc * 27 * eb + 16, 128) + 16;
    auto try_tile = [&](int TH, int TW, bool force_full, int budget, HaloPlan *p) {
        TH = TH < g.Ho ? TH : g.Ho;
        TW = TW < g.Wo ? TW : g.Wo;
        int HR = (TH - 1) * g.sh + (g.kh - 1) * g.dh + 2 * R + 2;
        int HC = (TW - 1) * g.sw + (g.kw - 1) * g.dw + 2 * R + 2;
        int full_h = force_full || HR >= g.H + 2;
        int full_w = force_full || HC >= g.W + 2;
        if (full_h) HR = g.H + 2;
        if (full_w) HC = g.W + 2;
        if (HR > 256 || HC > 256) return false;
        const long long halo = (long long)HR * HC * Gc * g.D * eb;
        const long long halo_r = (halo + 127) / 128 * 128;
        const long long total = halo_r + (long long)TH * TW * slot + 16;
        if (total > budget || total > smem_max) return false;
        *p = HaloPlan{TH, TW, Gc, R, HR, HC, full_h, full_w,
                      (g.Ho + TH - 1) / TH, (g.Wo + TW - 1) / TW, g.G / Gc,
                      slot, (int)halo_r, (int)total};
        return true;
    };
    static const int cands[][2] = {{16, 16}, {16, 8}, {8, 16}, {8, 8}, {8, 4}, {4, 8},
                                   {4, 4}, {4, 2}, {2, 4}, {2, 2}, {2, 1}, {1, 2}, {1, 1}};
    if (msdcn) {
        static const int big[][2] = {{32, 32}, {16, 32}, {32, 16}, {16, 16}, {8, 16}, {16, 8}, {8, 8}};
        for (auto &c : big)
            if (try_tile(c[0], c[1], true, smem_max, out)) return true;
    }
    for (int budget : {budget_two, smem_max})
        for (auto &c : cands)
            if (try_tile(c[0], c[1], false, budget, out)) return true;
    return false;
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

// Whether the halo kernel can run this call; fills plan and tensor map.
bool halo_ok(const Geometry &g, Dtype dt, bool msdcn, const void *in, const void *ow,
             const void *out, HaloPlan *plan, CUtensorMap *map) {
    const int eb = elem_bytes(dt);
    if (g.kh != 3 || g.kw != 3) return false;
    if ((g.D * eb) % 16 != 0) return false;
    const int U = g.D * eb / 16;
    if (U != 2 && U != 4 && U != 8) return false;
    if (!aligned16(in) || !aligned16(ow) || !aligned16(out)) return false;
    if (!plan_halo(g, eb, msdcn, plan)) return false;
    return encode_input_map(g, dt, in, *plan, map);
}

dcn4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DCN4_OK : DCN4_ERR_CUDA; }

dcn4_status run_forward(const dcn4_desc *desc, const void *input, const void *ow, void *output,
                        void *stream, const MsdcnParams *ms) {
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
    L.mixed = desc->math == DCN4_MATH_MIXED16;
    L.stream = static_cast<cudaStream_t>(stream);
    L.ow_bytes = (unsigned long long)g.N * g.Ho * g.Wo * g.G * g.K * 3 * elem_bytes(L.dtype);
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    if (desc->algo != DCN4_ALGO_GENERIC) {
        L.halo = halo_ok(g, L.dtype, L.msdcn, input, ow, output, &L.plan, &map);
        if (!L.halo && desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    }
    L.tmap = &map;
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

dcn4_status dcn4_backward_workspace_size(const dcn4_desc *desc, size_t *bytes) {
    Geometry g;
    if (!make_geometry(desc, &g) || !bytes) return DCN4_ERR_INVALID_ARG;
    *bytes = desc->dtype == DCN4_F32 ? 0 : (size_t)g.N * g.H * g.W * g.C * sizeof(float);
    return DCN4_OK;
}

dcn4_status dcn4_backward(const dcn4_desc *desc, const void *input, const void *offset_weight,
                          const void *grad_out, void *grad_input, void *grad_offset_weight,
                          void *workspace, size_t workspace_bytes, void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!input || !offset_weight || !grad_out || !grad_input || !grad_offset_weight)
        return DCN4_ERR_INVALID_ARG;
    size_t need = 0;
    dcn4_backward_workspace_size(desc, &need);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DCN4_ERR_WORKSPACE;
    if (desc->algo == DCN4_ALGO_HALO) return DCN4_ERR_UNSUPPORTED;
    BwdLaunch L;
    L.geo = g;
    L.dtype = static_cast<Dtype>(desc->dtype);
    L.in = input;
    L.ow = offset_weight;
    L.gout = grad_out;
    L.gin = grad_input;
    L.gow = grad_offset_weight;
    L.acc = need > 0 ? static_cast<float *>(workspace) : static_cast<float *>(grad_input);
    L.stream = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_backward(L));
}

dcn4_status msdcn_forward(const dcn4_desc *desc, const void *input, const void *dir_weight,
                          const void *scale_raw, const float *s0_host, float smax, void *output,
                          void *stream) {
    Geometry g;
    if (!make_geometry(desc, &g)) return DCN4_ERR_INVALID_ARG;
    if (!s0_host || !scale_raw) return DCN4_ERR_INVALID_ARG;
    static thread_local MsdcnParams ms;
    ms.raw = scale_raw;
    ms.smax = smax;
    for (int i = 0; i < g.G; ++i) ms.s0[i] = s0_host[i];
    return run_forward(desc, input, dir_weight, output, stream, &ms);
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

dcn4_status dcn4_last_device_error(unsigned int *code) {
    if (!code) return DCN4_ERR_INVALID_ARG;
    unsigned bits = 0;
    if (read_clear_device_error(&bits) != cudaSuccess) return DCN4_ERR_CUDA;
    *code = bits;
    if (bits & kErrTimeout) return DCN4_ERR_TIMEOUT;
    if (bits & kErrInternal) return DCN4_ERR_INTERNAL;
    return DCN4_OK;
}

}  // extern "C"
