// dcn4_producer.cuh -- the offset/weight producer of the DCNv4 module: a
// depthwise 3x3 convolution (stride 1, zero padding 1) of the feature map x
// followed by the single linear layer that emits all G*K*3 offsets and
// aggregation weights of a pixel ("(论文速读）DCNv4：高效可变形卷积算子",
// "方法3. DCN模块的微设计优化": with softmax gone the offset and weight
// projections merge into one linear layer, and the sub-network in front of it
// is a plain separable convolution).
//
//   h[p][c]   = dw_b[c] + sum_{i,j} dw_w[i][j][c] * x[p + (i-1, j-1)][c]
//   out[p][j] = lin_b[j] + sum_c lin_w[j][c] * h[p][c]
//
// Two kernels:
//  * producer_tc_kernel (16-bit data): one CTA per SM walks 128-pixel tiles.
//    Its warps compute h for the tile on the CUDA cores (fp32, rounded to the
//    data type, which is the operand type of the tensor cores) straight into
//    shared memory in the tcgen05 K-major core-matrix layout; one thread
//    issues the K/16 tcgen05.mma (M = 128 pixels, N = the outputs padded to
//    16, fp32 accumulators in tensor memory); all eight warps read the
//    accumulators back with tcgen05.ld, add the bias, round, and stage the
//    tile's rows, which leave in one bulk copy (the tile's outputs are
//    contiguous in global memory). lin_w stays resident in shared memory.
//  * producer_generic_kernel (any type and shape): 16 pixels per CTA, h in
//    shared memory (fp32, not rounded), the linear layer on the CUDA cores.
#pragma once

#include <type_traits>

#include "dcn4_common.cuh"

namespace dcn4 {

// ---------------------------------------------------------------------------
// tcgen05 helpers (cta_group::1)
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor, K-major, no swizzle: 8-row x 16-byte core
// matrices; `lbo` bytes between the two core matrices of one K = 16 step,
// `sbo` bytes between consecutive 8-row groups; descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_kmajor(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: fp32 accumulators, A and B of the same
// 16-bit type (bf16 when `bf16`, else fp16), both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16(bool bf16, int M, int N) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread t gets lane (base lane + t).
__device__ __forceinline__ void tc_ld_16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Bulk copy shared -> global (16-byte aligned addresses and size).
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 8 consecutive 16-bit values <-> fp32
template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const T *e = reinterpret_cast<const T *>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = Elem<T>::to_f(e[i]);
}
template <typename T>
__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 v;
    T *e = reinterpret_cast<T *>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) e[i] = Elem<T>::from_f(f[i]);
    return v;
}

// ---------------------------------------------------------------------------
// Tensor-core producer (bf16 / fp16)
// ---------------------------------------------------------------------------

// Byte offset of the 16-byte chunk q (channels 8q..8q+7) of row r in a
// K-major core-matrix tile whose rows hold C channels.
__device__ __forceinline__ uint32_t core_off(int r, int q, int C) {
    return (uint32_t)((r >> 3) * (C * 16) + q * 128 + (r & 7) * 16);
}

template <typename T>
__global__ void __launch_bounds__(256, 1)
    producer_tc_kernel(ProducerGeo pg, ProducerTcLayout L, const T *__restrict__ x,
                       const T *__restrict__ dw_w, const T *__restrict__ dw_b,
                       const T *__restrict__ lin_w, const T *__restrict__ lin_b,
                       T *__restrict__ out) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = pg.C, J = pg.J, NP = pg.NP, Q = C / 8;
    float *dwf = reinterpret_cast<float *>(smem + L.dwf_off);
    float *linb = reinterpret_cast<float *>(smem + L.linb_off);
    const uint32_t bar = smem_u32(smem + L.bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.bar_off + 8);

    // resident operands: lin_w in core-matrix layout (rows >= J zero), the
    // depthwise taps and both biases in fp32
    for (int i = tid; i < NP * Q; i += 256) {
        const int n = i / Q, q = i - n * Q;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < J) v = *reinterpret_cast<const uint4 *>(lin_w + (size_t)n * C + q * 8);
        *reinterpret_cast<uint4 *>(smem + L.b_off + core_off(n, q, C)) = v;
    }
    for (int i = tid; i < 9 * C; i += 256) dwf[i] = Elem<T>::to_f(dw_w[i]);
    for (int i = tid; i < C; i += 256) dwf[9 * C + i] = Elem<T>::to_f(dw_b[i]);
    for (int i = tid; i < NP; i += 256) linb[i] = i < J ? Elem<T>::to_f(lin_b[i]) : 0.f;
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(L.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = umma_idesc_f16(std::is_same<T, __nv_bfloat16>::value, 128, NP);
    const uint32_t a_base = smem_u32(smem + L.a_off), b_base = smem_u32(smem + L.b_off);
    const uint32_t s_base = smem_u32(smem + L.s_off);
    const int rlo = lane & 7, qlo = lane >> 3;
    const int qgroups = (Q + 3) / 4;
    bool ok = true;

    int iter = 0;
    for (int tile = blockIdx.x; tile < pg.ntiles; tile += gridDim.x, ++iter) {
        const long long p0 = (long long)tile * 128;
        const int rows = (int)min(128ll, pg.npix - p0);

        // depthwise 3x3 of the tile's pixels -> A (16-byte chunks; each
        // warp item covers 8 pixels x 4 chunks, conflict-free stores)
        for (int item = warp; item < 16 * qgroups; item += 8) {
            const int rg = item / qgroups, q = (item - rg * qgroups) * 4 + qlo;
            if (q >= Q) continue;
            const int r = rg * 8 + rlo;
            float acc[8];
            if (r < rows) {
                const long long p = p0 + r;
                const int xx = (int)(p % pg.W);
                const long long t = p / pg.W;
                const int y = (int)(t % pg.H);
                const int n = (int)(t / pg.H);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = dwf[9 * C + q * 8 + e];
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int yy = y + i - 1;
                    if (yy < 0 || yy >= pg.H) continue;
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        const int xs = xx + j - 1;
                        if (xs < 0 || xs >= pg.W) continue;
                        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
                            x + (((size_t)n * pg.H + yy) * pg.W + xs) * C + q * 8));
                        float f[8];
                        unpack8<T>(v, f);
                        const float *w = dwf + (i * 3 + j) * C + q * 8;
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[e], f[e], acc[e]);
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
            }
            *reinterpret_cast<uint4 *>(smem + L.a_off + core_off(r, q, C)) = pack8<T>(acc);
        }
        fence_async_smem();
        __syncthreads();

        // one thread issues the K/16 MMAs; the staging rows of the previous
        // tile must have left before the epilogue below rewrites them
        if (tid == 0) {
            bulk_wait_read();
            tc_fence_after();
            for (int kk = 0; kk < C / 16; ++kk)
                tc_mma_f16(tmem, umma_desc_kmajor(a_base + kk * 256, 128, C * 16),
                           umma_desc_kmajor(b_base + kk * 256, 128, C * 16), idesc, kk > 0);
            tc_commit(bar);
        }
        if (!mbar_wait_bounded(bar, iter & 1, kWaitLimitNs)) ok = false;
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // epilogue: warp w reads TMEM lanes 32 (w & 3) .. +31 (= tile rows),
        // 16-column chunks of parity w >> 2
        const int r = 32 * (warp & 3) + lane;
        for (int c16 = warp >> 2; c16 < NP / 16; c16 += 2) {
            float v[16];
            tc_ld_16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c16 * 16, v);
            const int c0 = c16 * 16;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (c0 + 8 * h >= J || r >= rows) continue;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = v[8 * h + e] + linb[c0 + 8 * h + e];
                *reinterpret_cast<uint4 *>(smem + L.s_off + ((size_t)r * J + c0 + 8 * h) * 2) =
                    pack8<T>(f);
            }
        }
        tc_fence_before();
        fence_async_smem();
        __syncthreads();
        if (tid == 0) bulk_store(out + p0 * J, s_base, (uint32_t)rows * J * 2);
    }

    if (tid == 0) {
        bulk_wait_all();
        if (!ok) atomicOr(&g_error_word, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(L.tmem_cols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Generic producer (any type, any C and J)
// ---------------------------------------------------------------------------

template <typename T>
__global__ void __launch_bounds__(256)
    producer_generic_kernel(ProducerGeo pg, const T *__restrict__ x, const T *__restrict__ dw_w,
                            const T *__restrict__ dw_b, const T *__restrict__ lin_w,
                            const T *__restrict__ lin_b, T *__restrict__ out) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float *h = reinterpret_cast<float *>(smem);  // [kProducerPixels][C]
    const int C = pg.C, J = pg.J;
    const long long p0 = (long long)blockIdx.x * kProducerPixels;
    const int rows = (int)min((long long)kProducerPixels, pg.npix - p0);
    for (int i = threadIdx.x; i < rows * C; i += blockDim.x) {
        const int r = i / C, c = i - r * C;
        const long long p = p0 + r;
        const int xx = (int)(p % pg.W);
        const long long t = p / pg.W;
        const int y = (int)(t % pg.H);
        const int n = (int)(t / pg.H);
        float acc = Elem<T>::to_f(dw_b[c]);
        for (int a = 0; a < 3; ++a) {
            const int yy = y + a - 1;
            if (yy < 0 || yy >= pg.H) continue;
            for (int b = 0; b < 3; ++b) {
                const int xs = xx + b - 1;
                if (xs < 0 || xs >= pg.W) continue;
                acc = fmaf(Elem<T>::to_f(dw_w[(a * 3 + b) * C + c]),
                           Elem<T>::to_f(x[(((size_t)n * pg.H + yy) * pg.W + xs) * C + c]), acc);
            }
        }
        h[i] = acc;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < rows * J; i += blockDim.x) {
        const int r = i / J, j = i - r * J;
        const T *wr = lin_w + (size_t)j * C;
        const float *hr = h + (size_t)r * C;
        float acc = Elem<T>::to_f(lin_b[j]);
        for (int c = 0; c < C; ++c) acc = fmaf(Elem<T>::to_f(wr[c]), hr[c], acc);
        out[(p0 + r) * J + j] = Elem<T>::from_f(acc);
    }
}

}  // namespace dcn4
