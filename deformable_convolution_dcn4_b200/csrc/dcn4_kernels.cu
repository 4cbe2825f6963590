// dcn4_kernels.cu -- the one translation unit holding every device function of
// libdcn4: kernel instantiations, their launchers and the device error word.
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "dcn4_common.cuh"

namespace dcn4 {
// Set by kernels whose bounded waits expire; read by dcn4_last_device_error.
__device__ unsigned int g_error_word = 0;

}  // namespace dcn4

#include "dcn4_bwd.cuh"
#include "dcn4_fwd.cuh"
#include "dcn4_bwd_halo.cuh"
#include "dcn4_bwd_vec.cuh"
#include "dcn4_producer.cuh"
#include "dcn4_launch.h"

namespace dcn4 {

namespace {

constexpr int kMaxDevices = 64;

// Kernel argument for launches without the multi-scale variant.
const MsdcnParams kNoMs = {};

// Kernels this library has issued (launched or captured into a graph).
std::atomic<unsigned long long> g_launches{0};
inline void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int cached_attr(cudaDeviceAttr attr, int (&cache)[kMaxDevices]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, attr, dev) == cudaSuccess) cache[dev] = v;
    }
    return cache[dev];
}

// Raises a kernel's dynamic shared memory limit once per (kernel, device) to
// the device's opt-in maximum minus the kernel's static shared memory.
cudaError_t allow_smem(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return cudaSuccess;
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, kernel);
    if (e != cudaSuccess) return e;
    const int limit = max_smem_optin() - (int)attr.sharedSizeBytes;
    if (bytes > limit) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
    if (e == cudaSuccess) done.insert({kernel, dev});
    return e;
}

int grid_for(long long work, int block) {
    long long blocks = (work + block - 1) / block;
    const long long cap = (long long)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

template <typename T, int U, bool MS, int MV, int STAGES, int NW>
cudaError_t launch_halo_t(const FwdLaunch &L) {
    auto k = fwd_halo_kernel<T, U, MS, MV, STAGES, NW>;
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
    k<<<(unsigned)grid, NT, L.plan.smem_bytes, L.stream>>>(
        *L.tmap, *L.tmap_ow, L.geo, L.plan, static_cast<const T *>(L.in),
        static_cast<const T *>(L.ow), static_cast<T *>(L.out), L.ow_bytes, L.ms ? *L.ms : kNoMs);
    count_launch();
    return cudaGetLastError();
}

// Stage count and warps: two stages with 16 warps when a tile has 512
// (pixel, group) pairs, 8 warps when it has fewer; the large single-stage
// plans (MSDCN whole-image windows, 64-channel groups) use 8.
template <typename T, int U, bool MS, int MV>
cudaError_t launch_halo_s(const FwdLaunch &L) {
    if constexpr (U <= 4) {
        if (L.plan.stages == 2) {
            if (L.plan.TH * L.plan.TW * L.plan.Gc >= 512)
                return launch_halo_t<T, U, MS, MV, 2, 16>(L);
            return launch_halo_t<T, U, MS, MV, 2, 8>(L);
        }
    }
    return launch_halo_t<T, U, MS, MV, 1, 8>(L);
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
            if (direct) return run(bwd_halo_kernel<T, 2, 8, true, true, MS>);
            return L.mixed ? run(bwd_halo_kernel<T, 2, 8, true, false, MS>)
                           : run(bwd_halo_kernel<T, 2, 8, false, false, MS>);
        }
        if (U == 2) {
            if (direct) return run(bwd_halo_kernel<T, 2, 16, true, true, MS>);
            return L.mixed ? run(bwd_halo_kernel<T, 2, 16, true, false, MS>)
                           : run(bwd_halo_kernel<T, 2, 16, false, false, MS>);
        }
    }
    if (U == 4 && nt == 256) return run(bwd_halo_kernel<T, 4, 8, false, false, MS>);
    if (U == 4) return run(bwd_halo_kernel<T, 4, 16, false, false, MS>);
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
    // 16-bit grad_input accumulates in place when the halo kernel runs in
    // the 16-bit weight mode; otherwise through the fp32 workspace
    const bool direct = L.halo && L.mixed && sizeof(T) == 2;
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

// One CTA whose barrier waits for 16 bytes that never come: the bounded wait
// expires and reports a timeout through the device error word.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_arrive_expect_tx(b, 16);
    const bool ok = mbar_wait_bounded(b, 0, limit_ns);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicOr(&g_error_word, kErrTimeout);
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream) {
    (void)cudaGetLastError();
    selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
    count_launch();
    return cudaGetLastError();
}

int sm_count() {
    static int cache[kMaxDevices] = {0};
    int v = cached_attr(cudaDevAttrMultiProcessorCount, cache);
    return v > 0 ? v : 148;
}

int max_smem_per_sm() {
    static int cache[kMaxDevices] = {0};
    int v = cached_attr(cudaDevAttrMaxSharedMemoryPerMultiprocessor, cache);
    return v > 0 ? v : 64 * 1024;
}

int max_smem_optin() {
    static int cache[kMaxDevices] = {0};
    int v = cached_attr(cudaDevAttrMaxSharedMemoryPerBlockOptin, cache);
    return v > 0 ? v : 48 * 1024;
}

cudaError_t launch_forward(const FwdLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::F32: return launch_fwd_t<float>(L);
        case Dtype::BF16: return launch_fwd_t<__nv_bfloat16>(L);
        case Dtype::F16: return launch_fwd_t<__half>(L);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_backward(const BwdLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::F32: return launch_bwd_t<float>(L);
        case Dtype::BF16: return launch_bwd_t<__nv_bfloat16>(L);
        case Dtype::F16: return launch_bwd_t<__half>(L);
    }
    return cudaErrorInvalidValue;
}

namespace {

template <typename T>
cudaError_t launch_producer_t(const ProducerLaunch &L) {
    const T *x = static_cast<const T *>(L.x), *dw_w = static_cast<const T *>(L.dw_w);
    const T *dw_b = static_cast<const T *>(L.dw_b), *lin_w = static_cast<const T *>(L.lin_w);
    const T *lin_b = static_cast<const T *>(L.lin_b);
    T *out = static_cast<T *>(L.out);
    if (L.tc) {
        if constexpr (sizeof(T) == 2) {
            const ProducerTcLayout &lay = L.lay;
            constexpr int NW = 16;  // measured: 16 warps 90 us, 8 warps 108 us (InternImage bf16)
            cudaError_t e = cudaFuncSetAttribute(producer_tc_kernel<T, NW>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 lay.bytes);
            if (e != cudaSuccess) return e;
            const int grid = L.pg.ntiles < sm_count() ? L.pg.ntiles : sm_count();
            producer_tc_kernel<T, NW><<<grid, NW * 32, lay.bytes, L.stream>>>(
                L.pg, lay, x, dw_w, dw_b, lin_w, lin_b, out);
            count_launch();
            return cudaGetLastError();
        }
        return cudaErrorInvalidValue;
    }
    const dim3 grid((unsigned)((L.pg.npix + kProducerPixels - 1) / kProducerPixels),
                    (unsigned)((L.pg.J + kProducerOuts - 1) / kProducerOuts));
    producer_generic_kernel<T><<<grid, 256, 0, L.stream>>>(L.pg, x, dw_w, dw_b, lin_w, lin_b, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_producer(const ProducerLaunch &L) {
    (void)cudaGetLastError();  // a pending error of an earlier call is not ours
    switch (L.dtype) {
        case Dtype::F32: return launch_producer_t<float>(L);
        case Dtype::BF16: return launch_producer_t<__nv_bfloat16>(L);
        case Dtype::F16: return launch_producer_t<__half>(L);
    }
    return cudaErrorInvalidValue;
}

cudaError_t read_clear_device_error(unsigned *bits) {
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

unsigned long long launches_issued() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace dcn4
