// dcn4_kernels_fused.cu -- the fused offset/weight producer + forward kernel
// of libdcn4 and its launcher.
#include "dcn4_common.cuh"

namespace dcn4 {
// Set by this unit's kernels when a bounded wait expires (one word per
// translation unit; read_clear_device_error ORs them).
static __device__ unsigned int g_error_word = 0;
}  // namespace dcn4

#include "dcn4_fused.cuh"
#include "dcn4_launch.h"

namespace dcn4 {

namespace {

// Kernel argument for the gathers, which never read it (no multi-scale).
const MsdcnParams kNoMs = {};

template <typename T, int U, int MV>
cudaError_t launch_fused_t(const FusedLaunch &L) {
    constexpr int NW = 16;
    auto k = fused_halo_kernel<T, U, MV, NW>;
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(k), L.lay.bytes);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, NW * 32, L.lay.bytes);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    // a multiple of the slice count, so that every CTA keeps one slice
    const long long units =
        (long long)L.geo.N * L.plan.tiles_h * L.plan.tiles_w * L.plan.slices;
    long long grid = (long long)sm_count() * occ;
    if (grid > units) grid = units;
    grid = grid / L.plan.slices * L.plan.slices;
    if (grid < L.plan.slices) grid = L.plan.slices;
    k<<<(unsigned)grid, NW * 32, L.lay.bytes, L.stream>>>(
        *L.tmap_in, *L.tmap_x, L.geo, L.plan, L.lay, static_cast<const T *>(L.in),
        static_cast<const T *>(L.dw_w), static_cast<const T *>(L.dw_b),
        static_cast<const T *>(L.lin_w), static_cast<const T *>(L.lin_b), static_cast<T *>(L.out),
        static_cast<T *>(L.rec_out), kNoMs, L.records_only ? 1 : 0);
    count_launch();
    return cudaGetLastError();
}

template <typename T, int U>
cudaError_t launch_fused_m(const FusedLaunch &L) {
    if (L.mathv == 2) return launch_fused_t<T, U, 2>(L);
    if (L.mathv == 1) return launch_fused_t<T, U, 1>(L);
    return launch_fused_t<T, U, 0>(L);
}

template <typename T>
cudaError_t launch_fused_u(const FusedLaunch &L) {
    const int U = L.geo.D * (int)sizeof(T) / 16;
    if (U == 2) return launch_fused_m<T, 2>(L);
    if (U == 4) return launch_fused_m<T, 4>(L);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_fused(const FusedLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::BF16: return launch_fused_u<__nv_bfloat16>(L);
        case Dtype::F16: return launch_fused_u<__half>(L);
        default: break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t read_clear_error_fused(unsigned *bits) {
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
