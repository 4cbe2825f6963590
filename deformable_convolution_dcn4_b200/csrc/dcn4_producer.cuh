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
// Three kernels:
//  * producer_tc2d_kernel (16-bit data, C a multiple of 64 up to 256, at most
//    256 outputs in whole 16-byte rows): 2-D pixel tiles, x by TMA tile load,
//    the sliding-window depthwise pass of depthwise_tile (shared with the
//    fused forward), one MMA over all outputs, rows written by one TMA tile
//    store (described at the kernel).
//  * producer_tc_kernel (16-bit data, the other tensor-core shapes): one CTA
//    per SM walks 128-pixel tiles
//    (128 consecutive pixels of the flattened N*H*W grid). The pixel range a
//    tile's 3x3 neighbourhoods touch (its pixels plus one image row and one
//    pixel on each side) arrives in one bulk copy, double-buffered so the
//    next tile's copy overlaps this tile's work. The warps compute h from
//    shared memory on the CUDA cores (fp32, rounded to the data type, the
//    operand type of the tensor cores) straight into the tcgen05 K-major
//    core-matrix layout; one thread issues the K/16 tcgen05.mma (M = 128
//    pixels, N = the outputs padded to 16, fp32 accumulators in tensor
//    memory); all warps read the accumulators back with tcgen05.ld, add the
//    bias and round; the tile's output rows are staged in its consumed input
//    buffer and leave in one bulk copy (else each thread stores 16-byte
//    pieces). lin_w stays resident in shared memory.
//  * producer_generic_kernel (any type and shape): 128 pixels x 128 outputs
//    per CTA, h (fp32, not rounded) and lin_w in channel chunks through
//    shared memory, 8 x 8 register blocks of outputs on the CUDA cores.
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

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base lane + t).
__device__ __forceinline__ void tc_ld_32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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

// acc[k] += w[k] * v[k] for eight 16-bit pairs: the sm_100 mixed-precision
// fma (16-bit multiplicands, exact product, one fp32 rounding), i.e. exactly
// fmaf on the widened values.
template <typename T> struct MixedFma8;
#define DCN4_MIXED_FMA8(TY, CT)                                                           \
    template <> struct MixedFma8<CT> {                                                    \
        static __device__ __forceinline__ void run(float *acc, const uint4 &v, const uint4 &w) { \
            const unsigned vv[4] = {v.x, v.y, v.z, v.w}, ww[4] = {w.x, w.y, w.z, w.w};    \
            _Pragma("unroll") for (int k = 0; k < 4; ++k) {                               \
                asm("{\n\t.reg .b16 vl, vh, wl, wh;\n\tmov.b32 {vl, vh}, %2;\n\t"          \
                    "mov.b32 {wl, wh}, %3;\n\tfma.rn.f32." TY " %0, vl, wl, %0;\n\t"          \
                    "fma.rn.f32." TY " %1, vh, wh, %1;\n\t}"                              \
                    : "+f"(acc[2 * k]), "+f"(acc[2 * k + 1])                              \
                    : "r"(vv[k]), "r"(ww[k]));                                            \
            }                                                                             \
        }                                                                                 \
    };
DCN4_MIXED_FMA8("bf16", __nv_bfloat16)
DCN4_MIXED_FMA8("f16", __half)
#undef DCN4_MIXED_FMA8

// ---------------------------------------------------------------------------
// Tensor-core producer (bf16 / fp16)
// ---------------------------------------------------------------------------

// Byte offset of the 16-byte chunk q (channels 8q..8q+7) of row r in a
// K-major core-matrix tile whose rows hold C channels.
__device__ __forceinline__ uint32_t core_off(int r, int q, int C) {
    return (uint32_t)((r >> 3) * (C * 16) + q * 128 + (r & 7) * 16);
}

// Depthwise 3x3 outputs of the tile's pixels (A row r = tile pixel
// ty*TW + tx) from the staged neighbourhood xs ((TH+2) x (TW+2) pixels of C
// values, the tile's top-left pixel at (1, 1)): bias, then the nine taps in
// row-major order as fp32 fma of the exact 16-bit products, rounded to T.
// Rows past the tile are left alone (zero since the CTA started).
// One item per thread: an 8-channel chunk q of one tile column tx over S
// consecutive rows. The item walks the S+2 staged rows it needs once, and
// each row's three vectors feed up to three output rows, so a staged vector
// is read (S+2)*3/S times per output row instead of 9, and the S*8
// accumulators give independent fma chains. C is a multiple of 64 (the
// host's plan: 128-byte staged pixels of whole groups). Eight consecutive
// items (one shared-memory phase) take 8 different chunks l = 0..7 of one
// block and columns (l + kx) mod TW: their staged reads hit 8 different
// bank quads (the pixel stride is a multiple of 128 bytes), and so do their
// core-matrix stores when TW >= 8.
template <typename T, int NW, int S>
__device__ __forceinline__ void depthwise_tile(const unsigned char *xs, unsigned char *a,
                                                const T *dwt, const float *dwb, int C, int TH,
                                                int TW, int lgTW, const unsigned char *sbase) {
    (void)sbase;
    constexpr int NT = NW * 32;
    const int XW = TW + 2;  // staged pixels per row
    const int PX = C * 2;   // bytes per staged pixel
    const int QB = C / 64;  // blocks of 8 chunks
    const int items = (TH + S - 1) / S * TW * QB * 8;
    for (int it = threadIdx.x; it < items; it += NT) {
        const int l = it & 7;
        int rest = it >> 3;
        const int qb = rest % QB;
        rest /= QB;
        const int kx = rest & (TW - 1), seg = rest >> lgTW;
        const int q = qb * 8 + l, tx = (l + kx) & (TW - 1), y0 = seg * S;
        const int ns = min(S, TH - y0);
        uint4 wv[9];
#pragma unroll
        for (int k = 0; k < 9; ++k) wv[k] = *reinterpret_cast<const uint4 *>(dwt + k * C + q * 8);
        const float4 *bb = reinterpret_cast<const float4 *>(dwb + q * 8);
        const float4 b0 = bb[0], b1 = bb[1];
        float acc[S][8];
#pragma unroll
        for (int y = 0; y < S; ++y) {
            acc[y][0] = b0.x, acc[y][1] = b0.y, acc[y][2] = b0.z, acc[y][3] = b0.w;
            acc[y][4] = b1.x, acc[y][5] = b1.y, acc[y][6] = b1.z, acc[y][7] = b1.w;
        }
        // staged row y0 + r, columns tx .. tx + 2 (tile rows y0 + r - 1)
        const unsigned char *col = xs + ((size_t)y0 * XW + tx) * PX + q * 16;
#pragma unroll
        for (int r = 0; r < S + 2; ++r) {
            if (r < ns + 2) {
                uint4 xv[3];
#pragma unroll
                for (int j = 0; j < 3; ++j) xv[j] = DCN4_LDS16(col + (r * XW + j) * PX, sbase);
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int y = r - i;  // output row fed by tap row i
                    if (y < 0 || y >= S) continue;
#pragma unroll
                    for (int j = 0; j < 3; ++j) MixedFma8<T>::run(acc[y], xv[j], wv[i * 3 + j]);
                }
            }
        }
#pragma unroll
        for (int y = 0; y < S; ++y) {
            if (y >= ns) continue;
            unsigned char *dst = a + core_off((y0 + y) * TW + tx, q, C);
            if (DCN4_SMEM_OK(dst, 16, sbase)) *reinterpret_cast<uint4 *>(dst) = pack8<T>(acc[y]);
        }
    }
}

template <typename T, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    producer_tc_kernel(ProducerGeo pg, ProducerTcLayout L, const T *__restrict__ x,
                       const T *__restrict__ dw_w, const T *__restrict__ dw_b,
                       const T *__restrict__ lin_w, const T *__restrict__ lin_b,
                       T *__restrict__ out) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = pg.C, J = pg.J, NP = pg.NP, Q = C / 8, W = pg.W;
    float *dwf = reinterpret_cast<float *>(smem + L.dwf_off);
    float *linb = reinterpret_cast<float *>(smem + L.linb_off);
    const uint32_t mma_bar = smem_u32(smem + L.bar_off);
    const uint32_t x_bar0 = mma_bar + 8;  // x_bar[b] at +8b
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.bar_off + 24);

    // resident operands: lin_w in core-matrix layout (rows >= J zero), the
    // depthwise taps and both biases in fp32
    constexpr int NT = NW * 32;
    // tensor extents (bounds of the checked build; unused otherwise)
    const unsigned long long x_b = (unsigned long long)pg.npix * C * 2;
    const unsigned long long out_b = (unsigned long long)pg.npix * J * 2;
    const unsigned long long lw_b = (unsigned long long)J * C * 2;
    (void)x_b, (void)out_b, (void)lw_b;
    for (int i = tid; i < NP * Q; i += NT) {
        const int n = i / Q, q = i - n * Q;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < J) v = DCN4_LDG16(lin_w + (size_t)n * C + q * 8, lin_w, lw_b);
        if (DCN4_SMEM_OK(smem + L.b_off + core_off(n, q, C), 16, smem))
            *reinterpret_cast<uint4 *>(smem + L.b_off + core_off(n, q, C)) = v;
    }
    T *dwt = reinterpret_cast<T *>(smem + L.dwt_off);  // dw_w [9][C] as stored
    if (DCN4_SMEM_OK(dwf, 10 * C * 4, smem) && DCN4_SMEM_OK(dwt, 9 * C * 2, smem) &&
        DCN4_SMEM_OK(linb, NP * 4, smem)) {
        for (int i = tid; i < 9 * C; i += NT) dwf[i] = Elem<T>::to_f(dw_w[i]);
        for (int i = tid; i < 9 * C; i += NT) dwt[i] = dw_w[i];
        for (int i = tid; i < C; i += NT) dwf[9 * C + i] = Elem<T>::to_f(dw_b[i]);
        for (int i = tid; i < NP; i += NT) linb[i] = i < J ? Elem<T>::to_f(lin_b[i]) : 0.f;
    }
    int2 *rowyx = reinterpret_cast<int2 *>(smem + L.row_off);  // (y, x) of each tile row

    // pixel rows a tile reads: its 128 pixels and one image row plus one
    // pixel on either side (clipped to the tensor), one contiguous range
    auto x_range = [&](int tile, long long &lo, long long &hi) {
        const long long p0 = (long long)tile * 128;
        lo = p0 - W - 1 > 0 ? p0 - W - 1 : 0;
        hi = p0 + 128 + W + 1 < pg.npix ? p0 + 128 + W + 1 : pg.npix;
    };
    int inflight = -1;  // (thread 0) buffer of a copy not yet waited for
    auto issue_x = [&](int tile, int b) {
        inflight = b;
        long long lo, hi;
        x_range(tile, lo, hi);
        const uint32_t bytes = (uint32_t)((hi - lo) * C * 2);
        mbar_arrive_expect_tx(x_bar0 + 8 * b, bytes);
        if (DCN4_CHECK(bytes <= (uint32_t)L.x_bytes) &&
            DCN4_SMEM_OK(smem + L.x_off + b * L.x_bytes, bytes, smem) &&
            DCN4_GMEM_OK(x + lo * C, bytes, x, x_b))
            bulk_load(smem_u32(smem + L.x_off + b * L.x_bytes), x + lo * C, bytes, x_bar0 + 8 * b);
    };
    if (tid == 0) {
        mbar_init(mma_bar, 1);
        mbar_init(x_bar0, 1);
        mbar_init(x_bar0 + 8, 1);
        fence_barrier_init();
        if ((int)blockIdx.x < pg.ntiles) issue_x(blockIdx.x, 0);
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
    // lane -> (row, chunk) of the depthwise pass. With whole 8-chunk blocks
    // the 8 lanes of each shared-memory phase take 8 different rows and 8
    // different chunks (a diagonal), so both the staged-pixel reads (pixel
    // stride a multiple of 128 bytes) and the core-matrix stores are free of
    // bank conflicts.
    const bool diag = Q % 8 == 0;
    const int e = lane & 7, f = lane >> 3;
    bool ok = true;

    int iter = 0;
    for (int tile = blockIdx.x; tile < pg.ntiles; tile += gridDim.x, ++iter) {
        const bool two = L.x_nbuf == 2;
        const int b = two ? iter & 1 : 0;
        const uint32_t x_par = two ? (iter >> 1) & 1 : iter & 1;
        const bool more = tile + (int)gridDim.x < pg.ntiles;
        const long long p0 = (long long)tile * 128;
        const int rows = (int)min(128ll, pg.npix - p0);
        long long lo, hi;
        x_range(tile, lo, hi);
        // two buffers: the other one was last read before the previous
        // tile's MMA
        if (two && tid == 0 && more) {
            bulk_wait_read();  // the previous tile's rows, staged in that buffer, have left
            issue_x(tile + gridDim.x, b ^ 1);
        }
        if (tid < 128 && DCN4_SMEM_OK(rowyx + tid, 8, smem)) {
            const int p = (int)p0 + tid;  // the pixel count fits an int
            const int t = p / W;
            rowyx[tid] = make_int2(t % pg.H, p - t * W);
        }
        if (!mbar_wait_bounded(x_bar0 + 8 * b, x_par, kWaitLimitNs)) ok = false;
        if (inflight == b) inflight = -1;
        const unsigned char *xs = smem + L.x_off + b * L.x_bytes;
        const int rel0 = (int)(p0 - lo);  // staged index of the tile's first pixel
        __syncthreads();

        // depthwise 3x3 of the tile's pixels -> A (fp32, rounded to T)
        auto dw_one = [&](int r, int q) {
            float acc[8];
            if (r < rows) {
                const int2 yx = rowyx[r];
                const int y = yx.x, xx = yx.y;
                const float4 *bb = reinterpret_cast<const float4 *>(dwf + 9 * C + q * 8);
                const float4 b0 = bb[0], b1 = bb[1];
                acc[0] = b0.x, acc[1] = b0.y, acc[2] = b0.z, acc[3] = b0.w;
                acc[4] = b1.x, acc[5] = b1.y, acc[6] = b1.z, acc[7] = b1.w;
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int yy = y + i - 1;
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        const int xj = xx + j - 1;
                        if (yy < 0 || yy >= pg.H || xj < 0 || xj >= W) continue;
                        const int idx = rel0 + r + (i - 1) * W + (j - 1);
                        const uint4 v = DCN4_LDS16(xs + idx * (C * 2) + q * 16, smem);
                        float fv[8];
                        unpack8<T>(v, fv);
                        const float4 *ww =
                            reinterpret_cast<const float4 *>(dwf + (i * 3 + j) * C + q * 8);
                        const float4 w0 = ww[0], w1 = ww[1];
                        acc[0] = fmaf(w0.x, fv[0], acc[0]);
                        acc[1] = fmaf(w0.y, fv[1], acc[1]);
                        acc[2] = fmaf(w0.z, fv[2], acc[2]);
                        acc[3] = fmaf(w0.w, fv[3], acc[3]);
                        acc[4] = fmaf(w1.x, fv[4], acc[4]);
                        acc[5] = fmaf(w1.y, fv[5], acc[5]);
                        acc[6] = fmaf(w1.z, fv[6], acc[6]);
                        acc[7] = fmaf(w1.w, fv[7], acc[7]);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[k] = 0.f;
            }
            if (DCN4_SMEM_OK(smem + L.a_off + core_off(r, q, C), 16, smem))
                *reinterpret_cast<uint4 *>(smem + L.a_off + core_off(r, q, C)) = pack8<T>(acc);
        };
        if (ok) {
            if (diag) {
                // blocks of 8 rows x 8 chunks; lane (e, f) keeps chunk
                // qb*8 + e and its 16-bit taps in registers and takes rows
                // (e + f + 4 s) & 7 of the block (mixed-precision fma: the
                // 16-bit products are exact, sums in fp32 as above)
                const int qblocks = Q / 8;
                for (int blk = warp; blk < 16 * qblocks; blk += NW) {
                    const int rb = blk / qblocks, q = (blk - rb * qblocks) * 8 + e;
                    uint4 wv[9];
#pragma unroll
                    for (int k = 0; k < 9; ++k)
                        wv[k] = *reinterpret_cast<const uint4 *>(dwt + k * C + q * 8);
                    const float4 *bb = reinterpret_cast<const float4 *>(dwf + 9 * C + q * 8);
                    const float4 b0 = bb[0], b1 = bb[1];
                    // the lane's two rows together: independent loads and
                    // fma chains in flight side by side
                    int rr[2];
                    int2 yx[2];
                    float acc[2][8];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        rr[s2] = rb * 8 + ((e + f + 4 * s2) & 7);
                        yx[s2] = rr[s2] < rows ? rowyx[rr[s2]] : make_int2(-1000000, 0);
                        acc[s2][0] = b0.x, acc[s2][1] = b0.y, acc[s2][2] = b0.z, acc[s2][3] = b0.w;
                        acc[s2][4] = b1.x, acc[s2][5] = b1.y, acc[s2][6] = b1.z, acc[s2][7] = b1.w;
                    }
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
#pragma unroll
                        for (int j = 0; j < 3; ++j) {
#pragma unroll
                            for (int s2 = 0; s2 < 2; ++s2) {
                                const int yy = yx[s2].x + i - 1, xj = yx[s2].y + j - 1;
                                if (yy < 0 || yy >= pg.H || xj < 0 || xj >= W) continue;
                                const int idx = rel0 + rr[s2] + (i - 1) * W + (j - 1);
                                const uint4 v = DCN4_LDS16(xs + idx * (C * 2) + q * 16, smem);
                                MixedFma8<T>::run(acc[s2], v, wv[i * 3 + j]);
                            }
                        }
                    }
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        if (rr[s2] >= rows) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) acc[s2][k] = 0.f;
                        }
                        if (DCN4_SMEM_OK(smem + L.a_off + core_off(rr[s2], q, C), 16, smem))
                            *reinterpret_cast<uint4 *>(smem + L.a_off + core_off(rr[s2], q, C)) =
                                pack8<T>(acc[s2]);
                    }
                }
            } else {
                for (int it = tid; it < 128 * Q; it += NT) {
                    const int r = it / Q;
                    dw_one(r, it - r * Q);
                }
            }
        }
        fence_async_smem();
        if (__syncthreads_or(!ok)) break;

        // one thread issues the K/16 MMAs (M = 128 pixels, N = NP outputs);
        // with one buffer the next tile's pixels start arriving now
        if (tid == 0) {
            if (!two && more) issue_x(tile + gridDim.x, 0);
            tc_fence_after();
            for (int kk = 0; kk < C / 16; ++kk)
                tc_mma_f16(tmem, umma_desc_kmajor(a_base + kk * 256, 128, C * 16),
                           umma_desc_kmajor(b_base + kk * 256, 128, C * 16), idesc, kk > 0);
            tc_commit(mma_bar);
        }
        if (!mbar_wait_bounded(mma_bar, iter & 1, kWaitLimitNs)) ok = false;
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // epilogue: warp w reads TMEM lanes 32 (w & 3) .. +31 (= tile rows),
        // every (NW / 4)-th 16-column chunk from w >> 2; bias, rounding.
        // With two input buffers the rows are staged in this tile's (now
        // consumed) buffer and leave in one bulk copy (the tile's outputs are
        // contiguous); else each thread stores its 16-byte pieces.
        const bool staged = two && L.x_bytes >= 128 * J * 2;
        unsigned char *srows = smem + L.x_off + b * L.x_bytes;
        const int r = 32 * (warp & 3) + lane;
        T *orow = out + (p0 + r) * J;
        for (int c16 = warp >> 2; c16 < NP / 16; c16 += NW / 4) {
            float v[16];
            tc_ld_16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c16 * 16, v);
            const int c0 = c16 * 16;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (c0 + 8 * h >= J || r >= rows) continue;
                float fo[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) fo[k] = v[8 * h + k] + linb[c0 + 8 * h + k];
                if (staged) {
                    if (DCN4_SMEM_OK(srows + ((size_t)r * J + c0 + 8 * h) * 2, 16, smem))
                        *reinterpret_cast<uint4 *>(srows + ((size_t)r * J + c0 + 8 * h) * 2) =
                            pack8<T>(fo);
                } else if (DCN4_GMEM_OK(orow + c0 + 8 * h, 16, out, out_b)) {
                    *reinterpret_cast<uint4 *>(orow + c0 + 8 * h) = pack8<T>(fo);
                }
            }
        }
        tc_fence_before();
        if (staged) fence_async_smem();
        __syncthreads();
        if (staged && tid == 0 && DCN4_SMEM_OK(srows, (unsigned)rows * J * 2, smem) &&
            DCN4_GMEM_OK(out + p0 * J, (unsigned)rows * J * 2, out, out_b))
            bulk_store(out + p0 * J, smem_u32(srows), (uint32_t)rows * J * 2);
    }
    if (tid == 0) bulk_wait_all();

    if (tid == 0 && !ok) {
        atomicOr(&g_error_word, kErrTimeout);
        // a prefetch issued before the failure lands before the CTA exits
        if (inflight >= 0)
            mbar_wait_bounded(x_bar0 + 8 * inflight,
                              L.x_nbuf == 2 ? ((iter + 1) >> 1) & 1 : (iter + 1) & 1, kWaitLimitNs);
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

// 2-D tiled tensor-core producer (bf16 / fp16, C a multiple of 64, J <= 256,
// whole 16-byte output rows): one CTA per SM walks TH x TW pixel tiles. Per
// tile, x's (TH+2) x (TW+2) neighbourhood arrives by one TMA tile load whose
// zero fill is the depthwise padding; the warps compute h with depthwise_tile
// (each staged vector read 4.5 times per output row instead of 9); one thread
// issues the C/16 MMAs (M = 128, N = NP, all J outputs) and the next tile's x
// load; the warps read the accumulators back, add the bias, round, and stage
// the tile's TH*TW rows of J values, which leave in one TMA tile store
// (columns and rows past the image are not written). Every wait is bounded.
template <typename T, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    producer_tc2d_kernel(const __grid_constant__ CUtensorMap tmap_x,
                         const __grid_constant__ CUtensorMap tmap_out, ProducerGeo pg,
                         ProducerTc2dLayout L, const T *__restrict__ dw_w,
                         const T *__restrict__ dw_b, const T *__restrict__ lin_w,
                         const T *__restrict__ lin_b) {
    extern __shared__ __align__(1024) unsigned char smem[];
    constexpr int NT = NW * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = pg.C, J = pg.J, NP = pg.NP, Q = C / 8;
    const int npx = L.TH * L.TW;
    const int ntiles = pg.N * L.tiles_h * L.tiles_w;
    unsigned char *xs = smem + L.x_off, *abuf = smem + L.a_off, *obuf = smem + L.o_off;
    T *dwt = reinterpret_cast<T *>(smem + L.dwt_off);
    float *dwb = reinterpret_cast<float *>(smem + L.dwb_off);
    float *linb = reinterpret_cast<float *>(smem + L.linb_off);
    const uint32_t x_bar = smem_u32(smem + L.bar_off), mma_bar = x_bar + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.bar_off + 16);
    const unsigned long long lw_b = (unsigned long long)J * C * 2;
    (void)lw_b;

    // resident operands; rows of h past the tile zero for good
    for (int i = tid; i < NP * Q; i += NT) {
        const int n = i / Q, q = i - n * Q;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < J) v = DCN4_LDG16(lin_w + (size_t)n * C + q * 8, lin_w, lw_b);
        if (DCN4_SMEM_OK(smem + L.b_off + core_off(n, q, C), 16, smem))
            *reinterpret_cast<uint4 *>(smem + L.b_off + core_off(n, q, C)) = v;
    }
    for (int i = npx * Q + tid; i < 128 * Q; i += NT) {
        const int r = i / Q, q = i - r * Q;
        if (DCN4_SMEM_OK(abuf + core_off(r, q, C), 16, smem))
            *reinterpret_cast<uint4 *>(abuf + core_off(r, q, C)) = make_uint4(0, 0, 0, 0);
    }
    if (DCN4_SMEM_OK(dwt, 9 * C * 2, smem) && DCN4_SMEM_OK(dwb, C * 4, smem) &&
        DCN4_SMEM_OK(linb, NP * 4, smem)) {
        for (int i = tid; i < 9 * C; i += NT) dwt[i] = dw_w[i];
        for (int i = tid; i < C; i += NT) dwb[i] = Elem<T>::to_f(dw_b[i]);
        for (int i = tid; i < NP; i += NT) linb[i] = i < J ? Elem<T>::to_f(lin_b[i]) : 0.f;
    }
    if (tid == 0) {
        mbar_init(x_bar, 1);
        mbar_init(mma_bar, 1);
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
    const uint32_t a_base = smem_u32(abuf), b_base = smem_u32(smem + L.b_off);

    // tile t: image n, output rows ho0.., columns wo0..
    auto coord = [&](int t, int &n, int &ho0, int &wo0) {
        const int tw = t % L.tiles_w;
        t /= L.tiles_w;
        ho0 = (t % L.tiles_h) * L.TH;
        n = t / L.tiles_h;
        wo0 = tw * L.TW;
    };
    // thread 32 issues the x loads, thread 0 the MMAs and the stores (so the
    // next x load and the MMAs go out side by side); each counts its own, for
    // the drain on an expired wait
    constexpr int kXThread = 32;
    int x_issued = 0, x_done = 0, mma_issued = 0, mma_done = 0;
    auto issue_x = [&](int t) {
        int n, ho0, wo0;
        coord(t, n, ho0, wo0);
        fence_async_smem();
        mbar_arrive_expect_tx(x_bar, (uint32_t)L.x_bytes);
        if (DCN4_SMEM_OK(xs, (unsigned)L.x_bytes, smem))
            tma_load_4d(smem_u32(xs), &tmap_x, 0, wo0 - 1, ho0 - 1, n, x_bar);
        ++x_issued;
    };
    if (tid == kXThread && (int)blockIdx.x < ntiles) issue_x(blockIdx.x);

    bool ok = true;
    int k = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
        const uint32_t par = (uint32_t)k & 1u;
        if (!mbar_wait_bounded(x_bar, par, kWaitLimitNs)) ok = false;
        else if (tid == kXThread) ++x_done;
        if (__syncthreads_or(!ok)) break;
        depthwise_tile<T, NW, 4>(xs, abuf, dwt, dwb, C, L.TH, L.TW, L.lgTW, smem);
        fence_async_smem();
        __syncthreads();
        if (tid == kXThread && t + (int)gridDim.x < ntiles) issue_x(t + gridDim.x);
        if (tid == 0) {
            tc_fence_after();
            for (int kk = 0; kk < C / 16; ++kk)
                tc_mma_f16(tmem, umma_desc_kmajor(a_base + kk * 256, 128, C * 16),
                           umma_desc_kmajor(b_base + kk * 256, 128, C * 16), idesc, kk > 0);
            tc_commit(mma_bar);
            ++mma_issued;
            bulk_wait_read();  // the previous tile's store has read the staged rows
        }
        if (!mbar_wait_bounded(mma_bar, par, kWaitLimitNs)) ok = false;
        else if (tid == 0) ++mma_done;
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();

        // accumulators -> staged rows (row stride J*2 bytes, a multiple of 16):
        // 32-column reads (one wait each), a 16-column tail when NP % 32 != 0
        const int r = 32 * (warp & 3) + lane;
        const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        auto stage8 = [&](const float *v, int c0) {
            if (r >= npx || c0 >= J) return;
            float fo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) fo[e] = v[e] + linb[c0 + e];
            unsigned char *dst = obuf + (size_t)r * J * 2 + c0 * 2;
            if (DCN4_SMEM_OK(dst, 16, smem)) *reinterpret_cast<uint4 *>(dst) = pack8<T>(fo);
        };
        for (int c32 = warp >> 2; c32 < NP / 32; c32 += NW / 4) {
            float v[32];
            tc_ld_32(trow + c32 * 32, v);
#pragma unroll
            for (int h = 0; h < 4; ++h) stage8(v + 8 * h, c32 * 32 + 8 * h);
        }
        if ((NP & 16) && (warp >> 2) == (NP / 32) % (NW / 4)) {
            float v[16];
            tc_ld_16(trow + (NP / 32) * 32, v);
            stage8(v, (NP / 32) * 32);
            stage8(v + 8, (NP / 32) * 32 + 8);
        }
        tc_fence_before();
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            int n, ho0, wo0;
            coord(t, n, ho0, wo0);
            if (DCN4_SMEM_OK(obuf, (unsigned)npx * J * 2, smem))
                tma_store_4d(&tmap_out, smem_u32(obuf), 0, wo0, ho0, n);
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == kXThread && !ok && x_issued > x_done)
        mbar_wait_bounded(x_bar, (uint32_t)(x_issued - 1) & 1u, kWaitLimitNs);
    if (tid == 0 && !ok) {
        atomicOr(&g_error_word, kErrTimeout);
        if (mma_issued > mma_done)
            mbar_wait_bounded(mma_bar, (uint32_t)(mma_issued - 1) & 1u, kWaitLimitNs);
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

// Tile of kProducerPixels pixels x kProducerOuts outputs per 256-thread
// CTA; K (= C) in chunks of kProducerK channels: the chunk's depthwise
// outputs h (fp32) and the chunk of lin_w go to shared memory, k-major, and
// each thread accumulates an 8 x 8 block of outputs in registers.
template <typename T>
__global__ void __launch_bounds__(256, 2)
    producer_generic_kernel(ProducerGeo pg, const T *__restrict__ x, const T *__restrict__ dw_w,
                            const T *__restrict__ dw_b, const T *__restrict__ lin_w,
                            const T *__restrict__ lin_b, T *__restrict__ out) {
    constexpr int PM = kProducerPixels, PN = kProducerOuts, KC = kProducerK, LD = PM + 4;
    static_assert(PM == 128 && PN == 128, "16 x 16 threads of 8 x 8 outputs");
    __shared__ __align__(16) float hs[KC][LD];  // h chunk, [k][pixel]
    __shared__ __align__(16) float ws[KC][LD];  // lin_w chunk, [k][output]
    __shared__ int2 rowyx[PM];                  // (image row index n*H + y, x) per pixel
    const int C = pg.C, J = pg.J, tid = threadIdx.x;
    const long long p0 = (long long)blockIdx.x * PM;
    const int j0 = blockIdx.y * PN;
    const int rows = (int)min((long long)PM, pg.npix - p0);
    if (tid < PM) {
        const long long p = p0 + tid;
        rowyx[tid] = make_int2((int)(p / pg.W), (int)(p % pg.W));
    }
    const int tx = tid & 15, ty = tid >> 4;  // outputs 8tx.., pixels 8ty..
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
    __syncthreads();
    for (int c0 = 0; c0 < C; c0 += KC) {
        // depthwise outputs of the chunk: lanes over channels (coalesced)
        for (int i = tid; i < PM * KC; i += 256) {
            const int r = i / KC, k = i - r * KC, c = c0 + k;
            float v = 0.f;
            if (r < rows && c < C) {
                const int ny = rowyx[r].x, xx = rowyx[r].y, y = ny % pg.H;
                v = Elem<T>::to_f(dw_b[c]);
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    const int yy = y + a - 1;
                    if (yy < 0 || yy >= pg.H) continue;
#pragma unroll
                    for (int b = 0; b < 3; ++b) {
                        const int xs = xx + b - 1;
                        if (xs < 0 || xs >= pg.W) continue;
                        const T *xp = x + ((size_t)(ny + a - 1) * pg.W + xs) * C + c;
                        if (!DCN4_GMEM_OK(xp, sizeof(T), x,
                                          (unsigned long long)pg.npix * C * sizeof(T)))
                            continue;
                        v = fmaf(Elem<T>::to_f(dw_w[(a * 3 + b) * C + c]), Elem<T>::to_f(*xp), v);
                    }
                }
            }
            hs[k][r] = v;
        }
        // the chunk of lin_w: lanes over channels (coalesced)
        for (int i = tid; i < PN * KC; i += 256) {
            const int jj = i / KC, k = i - jj * KC, j = j0 + jj, c = c0 + k;
            ws[k][jj] = (j < J && c < C) ? Elem<T>::to_f(lin_w[(size_t)j * C + c]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < KC; ++k) {
            const float4 h0 = *reinterpret_cast<const float4 *>(&hs[k][8 * ty]);
            const float4 h1 = *reinterpret_cast<const float4 *>(&hs[k][8 * ty + 4]);
            const float4 w0 = *reinterpret_cast<const float4 *>(&ws[k][8 * tx]);
            const float4 w1 = *reinterpret_cast<const float4 *>(&ws[k][8 * tx + 4]);
            const float h8[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            const float w8[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(h8[a], w8[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int r = 8 * ty + a;
        if (r >= rows) continue;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int j = j0 + 8 * tx + b;
            if (j < J && DCN4_GMEM_OK(out + (p0 + r) * J + j, sizeof(T), out,
                                      (unsigned long long)pg.npix * J * sizeof(T)))
                out[(p0 + r) * J + j] = Elem<T>::from_f(acc[a][b] + Elem<T>::to_f(lin_b[j]));
        }
    }
}

}  // namespace dcn4
