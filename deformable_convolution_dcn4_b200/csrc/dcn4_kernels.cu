// dcn4_kernels.cu -- the offset/weight producer and the bounded-wait
// self-test kernels with their launchers, plus the host helpers every kernel
// unit shares (device attributes, shared-memory opt-in, grid sizing, the
// launch counter, the device error words).
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "dcn4_common.cuh"

namespace dcn4 {
// Set by this unit's kernels when a bounded wait expires (one word per
// translation unit; read_clear_device_error ORs them).
static __device__ unsigned int g_error_word = 0;
}  // namespace dcn4

#include "dcn4_producer.cuh"
#include "dcn4_launch.h"

namespace dcn4 {

namespace {

constexpr int kMaxDevices = 64;

// Kernels this library has issued (launched or captured into a graph).
std::atomic<unsigned long long> g_launches{0};

int cached_attr(cudaDeviceAttr attr, int (&cache)[kMaxDevices]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, attr, dev) == cudaSuccess) cache[dev] = v;
    }
    return cache[dev];
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

template <typename T>
cudaError_t launch_producer_t(const ProducerLaunch &L) {
    const T *x = static_cast<const T *>(L.x), *dw_w = static_cast<const T *>(L.dw_w);
    const T *dw_b = static_cast<const T *>(L.dw_b), *lin_w = static_cast<const T *>(L.lin_w);
    const T *lin_b = static_cast<const T *>(L.lin_b);
    T *out = static_cast<T *>(L.out);
    if (L.tc2d) {
        if constexpr (sizeof(T) == 2) {
            constexpr int NW = 16;
            auto k = producer_tc2d_kernel<T, NW>;
            cudaError_t e = allow_smem(reinterpret_cast<const void *>(k), L.lay2.bytes);
            if (e != cudaSuccess) return e;
            const int tiles = L.pg.N * L.lay2.tiles_h * L.lay2.tiles_w;
            const int grid = tiles < sm_count() ? tiles : sm_count();
            k<<<grid, NW * 32, L.lay2.bytes, L.stream>>>(*L.tmap_x, *L.tmap_out, L.pg, L.lay2,
                                                        dw_w, dw_b, lin_w, lin_b);
            count_launch();
            return cudaGetLastError();
        }
        return cudaErrorInvalidValue;
    }
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

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

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
    unsigned v = 0, f = 0, b = 0, u = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v));
    if (e != cudaSuccess) return e;
    if (v != 0) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return e;
    }
    e = read_clear_error_fwd(&f);
    if (e != cudaSuccess) return e;
    e = read_clear_error_bwd(&b);
    if (e != cudaSuccess) return e;
    e = read_clear_error_fused(&u);
    if (e != cudaSuccess) return e;
    *bits = v | f | b | u;
    return cudaSuccess;
}

unsigned long long launches_issued() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace dcn4
