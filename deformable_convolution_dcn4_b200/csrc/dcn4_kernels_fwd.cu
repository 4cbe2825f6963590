// dcn4_kernels_fwd.cu -- forward kernels of libdcn4 (staged halo, vectorised
// and scalar global-memory, DCNv4 and MSDCN) and their launcher.
#include <cstring>

#include "dcn4_common.cuh"

namespace dcn4 {
// Set by this unit's kernels when a bounded wait expires (one word per
// translation unit; read_clear_device_error ORs them).
static __device__ unsigned int g_error_word = 0;
}  // namespace dcn4

#include "dcn4_fwd.cuh"
#include "dcn4_bwd_vec.cuh"
#include "dcn4_launch.h"

namespace dcn4 {

namespace {

// Kernel argument for launches without the multi-scale variant.
const MsdcnParams kNoMs = {};

template <typename T, int U, bool MS, int MV, int STAGES, int NW, int LPP = 1>
cudaError_t launch_halo_t(const FwdLaunch &L) {
    auto k = fwd_halo_kernel<T, U, MS, MV, STAGES, NW, LPP>;
    constexpr int NT = NW * 32;
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(k), L.plan.smem_bytes);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)L.geo.N * L.plan.slices * L.plan.tiles_h * L.plan.tiles_w;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, NT, L.plan.smem_bytes);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    long long grid = (long long)sm_count() * occ;
    if (grid > tiles) grid = tiles;
    // deferred escapes: each CTA's region of entries
    EscList el;
    memset(&el, 0, sizeof(el));
    if constexpr (LPP == 1) {
        const size_t entry = escape_entry_bytes(L.geo.D, (int)sizeof(T));
        if (L.ws != nullptr && L.ws_bytes >= entry * (size_t)grid) {
            size_t cap = L.ws_bytes / entry / (size_t)grid;
            if (cap > (size_t)(1 << 30)) cap = (size_t)1 << 30;
            el.entries = static_cast<unsigned char *>(L.ws);
            el.cap = (int)cap;
            el.entry_bytes = (int)entry;
            el.bytes = (unsigned long long)(cap * entry * (size_t)grid);
        }
    }
    k<<<(unsigned)grid, NT, L.plan.smem_bytes, L.stream>>>(
        *L.tmap, *L.tmap_ow, L.geo, L.plan, static_cast<const T *>(L.in),
        static_cast<const T *>(L.ow), static_cast<T *>(L.out), L.ow_bytes, L.ms ? *L.ms : kNoMs,
        el);
    count_launch();
    e = cudaGetLastError();
    return e;
}

// Stage count and warps: two stages with 16 warps when a tile has 512
// (pixel, group) pairs, 8 warps when it has fewer; the large single-stage
// plans (MSDCN whole-image windows) use 8, and groups of 8 chunks (64 bf16 /
// 32 fp32 channels) run two lanes per pair on 16 warps.
template <typename T, int U, bool MS, int MV>
cudaError_t launch_halo_s(const FwdLaunch &L) {
    if constexpr (U <= 4) {
        if (L.plan.stages == 2) {
            if (L.plan.TH * L.plan.TW * L.plan.Gc >= 512)
                return launch_halo_t<T, U, MS, MV, 2, 16>(L);
            return launch_halo_t<T, U, MS, MV, 2, 8>(L);
        }
        return launch_halo_t<T, U, MS, MV, 1, 8>(L);
    } else {
        return launch_halo_t<T, U, MS, MV, 1, 16, 2>(L);
    }
}

template <typename T, int U, bool MS>
cudaError_t launch_halo_m(const FwdLaunch &L) {
    if constexpr (sizeof(T) == 2) {
        if (L.mathv == 2) return launch_halo_s<T, U, MS, 2>(L);
        if (L.mathv == 1) return launch_halo_s<T, U, MS, 1>(L);
    }
    return launch_halo_s<T, U, MS, 0>(L);
}

template <typename T, bool MS>
cudaError_t launch_halo_u(const FwdLaunch &L) {
    const int U = L.geo.D * (int)sizeof(T) / 16;
    if constexpr (sizeof(T) == 2) {
        if (U == 2) return launch_halo_m<T, 2, MS>(L);
    }
    if (U == 4) return launch_halo_m<T, 4, MS>(L);
    if (U == 8) return launch_halo_m<T, 8, MS>(L);
    return cudaErrorInvalidValue;
}

template <typename T, bool MS>
cudaError_t launch_generic_t(const FwdLaunch &L) {
    const long long work = (long long)L.geo.N * L.geo.Ho * L.geo.Wo * L.geo.G * ((L.geo.D + 7) / 8);
    fwd_generic_kernel<T, MS><<<grid_for(work, 256), 256, 0, L.stream>>>(
        L.geo, static_cast<const T *>(L.in), static_cast<const T *>(L.ow), static_cast<T *>(L.out),
        L.ms ? *L.ms : kNoMs);
    count_launch();
    return cudaGetLastError();
}

template <typename T, bool MS>
cudaError_t launch_fwd_vec_t(const FwdLaunch &L) {
    const long long work = (long long)L.geo.N * L.geo.Ho * L.geo.Wo * L.geo.G *
                           (L.geo.D / Elem<T>::kPerVec);
    fwd_vec_kernel<T, MS><<<grid_for(work, 256), 256, 0, L.stream>>>(
        L.geo, static_cast<const T *>(L.in), static_cast<const T *>(L.ow), static_cast<T *>(L.out),
        L.ms ? *L.ms : kNoMs);
    count_launch();
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fwd_t(const FwdLaunch &L) {
    if (L.halo) return L.msdcn ? launch_halo_u<T, true>(L) : launch_halo_u<T, false>(L);
    if (L.vec) return L.msdcn ? launch_fwd_vec_t<T, true>(L) : launch_fwd_vec_t<T, false>(L);
    return L.msdcn ? launch_generic_t<T, true>(L) : launch_generic_t<T, false>(L);
}

}  // namespace

cudaError_t launch_forward(const FwdLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::F32: return launch_fwd_t<float>(L);
        case Dtype::BF16: return launch_fwd_t<__nv_bfloat16>(L);
        case Dtype::F16: return launch_fwd_t<__half>(L);
    }
    return cudaErrorInvalidValue;
}

size_t escape_entry_bytes(int D, int eb) {
    (void)eb;
    return 16 + 4 * (size_t)D;
}

size_t forward_escape_bytes(long long npairs, int D, int eb, int ctas) {
    return (size_t)((npairs + 3) / 4 + ctas) * escape_entry_bytes(D, eb);
}

cudaError_t read_clear_error_fwd(unsigned *bits) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v));
    if (e != cudaSuccess) return e;
    if (v != 0) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    }
    *bits = v;
    return e;
}

}  // namespace dcn4
