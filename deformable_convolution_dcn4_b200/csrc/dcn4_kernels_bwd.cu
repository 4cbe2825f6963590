// dcn4_kernels_bwd.cu -- backward kernels of libdcn4 (staged halo,
// vectorised and scalar global-memory, DCNv4 and MSDCN; zero and convert
// passes) and their launcher.
#include "dcn4_common.cuh"

namespace dcn4 {
// Set by this unit's kernels when a bounded wait expires (one word per
// translation unit; read_clear_device_error ORs them).
static __device__ unsigned int g_error_word = 0;
}  // namespace dcn4

#include "dcn4_bwd.cuh"
#include "dcn4_fwd.cuh"
#include "dcn4_bwd_halo.cuh"
#include "dcn4_bwd_vec.cuh"
#include "dcn4_launch.h"

namespace dcn4 {

namespace {

// Kernel argument for launches without the multi-scale variant.
const MsdcnParams kNoMs = {};

template <typename T, bool MS>
cudaError_t launch_bwd_halo_m(const BwdLaunch &L, bool direct) {
    const int U = L.geo.D * (int)sizeof(T) / 16;
    const long long grid = (long long)L.geo.N * L.plan.slices * L.plan.tiles_h * L.plan.tiles_w;
    const int nt = L.layout.threads;
    auto run = [&](auto kernel) {
        cudaError_t e = allow_smem(reinterpret_cast<const void *>(kernel), L.layout.smem_bytes);
        if (e != cudaSuccess) return e;
        kernel<<<(unsigned)grid, nt, L.layout.smem_bytes, L.stream>>>(
            *L.tmap_in, *L.tmap_go, *L.tmap_ow, L.geo, L.plan, L.layout, static_cast<const T *>(L.in),
            static_cast<const T *>(L.ow), static_cast<T *>(L.gow), L.acc, static_cast<T *>(L.gin),
            L.ow_bytes, L.ms ? *L.ms : kNoMs, static_cast<T *>(L.graw));
        count_launch();
        return cudaGetLastError();
    };
    if constexpr (sizeof(T) == 2) {
        if (U == 2 && nt == 256) {
            if (direct) return run(bwd_halo_kernel<T, 2, 8, true, true, MS, 1>);
            return L.mixed ? run(bwd_halo_kernel<T, 2, 8, true, false, MS, 1>)
                           : run(bwd_halo_kernel<T, 2, 8, false, false, MS, 1>);
        }
        if (U == 2) {
            if (direct) return run(bwd_halo_kernel<T, 2, 16, true, true, MS, 1>);
            return L.mixed ? run(bwd_halo_kernel<T, 2, 16, true, false, MS, 1>)
                           : run(bwd_halo_kernel<T, 2, 16, false, false, MS, 1>);
        }
        // 64 channels: four lanes per (pixel, group), 256 or 512 threads
        if (U == 8 && L.layout.lpp == 4 && nt == 256) {
            if (direct) return run(bwd_halo_kernel<T, 8, 8, true, true, MS, 4>);
            return L.mixed ? run(bwd_halo_kernel<T, 8, 8, true, false, MS, 4>)
                           : run(bwd_halo_kernel<T, 8, 8, false, false, MS, 4>);
        }
        if (U == 8 && L.layout.lpp == 4) {
            if (direct) return run(bwd_halo_kernel<T, 8, 16, true, true, MS, 4>);
            return L.mixed ? run(bwd_halo_kernel<T, 8, 16, true, false, MS, 4>)
                           : run(bwd_halo_kernel<T, 8, 16, false, false, MS, 4>);
        }
    } else {
        // fp32, 32 channels: four lanes per (pixel, group), 256 or 512 threads
        if (U == 8 && L.layout.lpp == 4 && nt == 256)
            return run(bwd_halo_kernel<T, 8, 8, false, false, MS, 4>);
        if (U == 8 && L.layout.lpp == 4) return run(bwd_halo_kernel<T, 8, 16, false, false, MS, 4>);
    }
    if (U == 4 && nt == 256) return run(bwd_halo_kernel<T, 4, 8, false, false, MS, 1>);
    if (U == 4) return run(bwd_halo_kernel<T, 4, 16, false, false, MS, 1>);
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_bwd_halo(const BwdLaunch &L, bool direct) {
    return L.msdcn ? launch_bwd_halo_m<T, true>(L, direct) : launch_bwd_halo_m<T, false>(L, direct);
}

template <typename T, bool MS, int LPP>
cudaError_t launch_bwd_vec_l(const BwdLaunch &L) {
    const Geometry &g = L.geo;
    const long long total = (long long)g.N * g.Ho * g.Wo * g.G * LPP;
    bwd_vec_kernel<T, MS, LPP><<<grid_for(total, 256), 256, 0, L.stream>>>(
        g, static_cast<const T *>(L.in), static_cast<const T *>(L.ow),
        static_cast<const T *>(L.gout), L.acc, static_cast<T *>(L.gow), L.ms ? *L.ms : kNoMs,
        static_cast<T *>(L.graw));
    count_launch();
    return cudaGetLastError();
}

template <typename T, bool MS>
cudaError_t launch_bwd_vec_m(const BwdLaunch &L) {
    switch (L.geo.D * (int)sizeof(T) / 16) {
        case 1: return launch_bwd_vec_l<T, MS, 1>(L);
        case 2: return launch_bwd_vec_l<T, MS, 2>(L);
        case 4: return launch_bwd_vec_l<T, MS, 4>(L);
        case 8: return launch_bwd_vec_l<T, MS, 8>(L);
        case 16: return launch_bwd_vec_l<T, MS, 16>(L);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_bwd_vec(const BwdLaunch &L) {
    return L.msdcn ? launch_bwd_vec_m<T, true>(L) : launch_bwd_vec_m<T, false>(L);
}

template <typename T>
cudaError_t launch_bwd_t(const BwdLaunch &L) {
    const Geometry &g = L.geo;
    const long long nin = (long long)g.N * g.H * g.W * g.C;
    // 16-bit grad_input accumulates in place when the caller asked for
    // 16-bit cross-CTA accumulation and the halo kernel runs; otherwise
    // through the fp32 workspace (zeroed, then converted once)
    const bool direct = L.halo && L.mixed && L.acc16 && sizeof(T) == 2;
    cudaError_t e;
    if (direct) {
        zero_bytes_kernel<<<grid_for(nin * (long long)sizeof(T) / 16 + 1, 256), 256, 0, L.stream>>>(
            static_cast<unsigned char *>(L.gin), nin * (long long)sizeof(T));
        count_launch();
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_bwd_halo<T>(L, true);
    }
    zero_f32_kernel<<<grid_for(nin / 4 + 1, 256), 256, 0, L.stream>>>(L.acc, nin);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.halo) {
        e = launch_bwd_halo<T>(L, false);
    } else if (L.vec) {
        e = launch_bwd_vec<T>(L);
    } else {
        const long long pairs = (long long)g.N * g.Ho * g.Wo * g.G;
        if (L.msdcn)
            bwd_generic_kernel<T, true><<<grid_for(pairs, 256), 256, 0, L.stream>>>(
                g, static_cast<const T *>(L.in), static_cast<const T *>(L.ow),
                static_cast<const T *>(L.gout), L.acc, static_cast<T *>(L.gow), *L.ms,
                static_cast<T *>(L.graw));
        else
            bwd_generic_kernel<T, false><<<grid_for(pairs, 256), 256, 0, L.stream>>>(
                g, static_cast<const T *>(L.in), static_cast<const T *>(L.ow),
                static_cast<const T *>(L.gout), L.acc, static_cast<T *>(L.gow), kNoMs, nullptr);
        count_launch();
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if (static_cast<void *>(L.acc) != L.gin) {
        convert_f32_kernel<T><<<grid_for(nin / 4 + 1, 256), 256, 0, L.stream>>>(
            L.acc, static_cast<T *>(L.gin), nin);
        count_launch();
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

cudaError_t launch_backward(const BwdLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::F32: return launch_bwd_t<float>(L);
        case Dtype::BF16: return launch_bwd_t<__nv_bfloat16>(L);
        case Dtype::F16: return launch_bwd_t<__half>(L);
    }
    return cudaErrorInvalidValue;
}

cudaError_t read_clear_error_bwd(unsigned *bits) {
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
