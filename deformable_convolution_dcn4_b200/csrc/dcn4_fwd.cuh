// dcn4_fwd.cuh -- forward kernels of DCNv4 and its groupwise multi-scale
// variant (MSDCN).
//
// Operation (DCNv4 paper digest "(论文速读）DCNv4：高效可变形卷积算子", sections
// "移除Softmax归一化" and "方法1. 消除冗余工作负载"; FlowDCN article "2.2 DCN结构简介"
// and "3.1 组间多尺度可变形卷积"): out[p0, g*D + d] = sum_k m_k * bilinear(in, p0 +
// p_k + dp_k)[g*D + d], with the D channels of a group sharing the offsets and
// weights, and for MSDCN dp_k = s_g(p0) * dir_k.
//
// Two kernels:
//  * fwd_generic_kernel: one thread per (pixel, group, run of <= 8 channels),
//    scalar loads straight from global memory. Any shape, any alignment.
//  * fwd_halo_kernel: one thread per (pixel, group) covering all D channels.
//    A CTA owns an output tile x a slice of Gc groups. One TMA tile load
//    brings the input window the tile can reach (tile +- R pixels, zeros
//    outside the image by the TMA out-of-bounds fill) into shared memory, and
//    bulk copies bring the tile's offset/weight records. Every corner gather
//    is then a 16-byte shared-memory load; samples that leave the window use
//    16-byte global loads instead. Lanes rotate the order of their 16-byte
//    chunks so that the 8 lanes of each shared-memory phase hit 8 different
//    bank quads whatever pixel they sample (the pixel stride is a multiple of
//    128 bytes), which keeps random gathers free of bank conflicts.
#pragma once

#include "dcn4_common.cuh"

namespace dcn4 {

// The device error word (defined once, in dcn4_kernels.cu, before this file).

// s = min(s0 * softplus(raw), smax), softplus(r) = max(r, 0) + log1p(exp(-|r|)).
__device__ __forceinline__ float msdcn_scale(float raw, float s0, float smax) {
    float sp = __fadd_rn(fmaxf(raw, 0.0f), log1pf(expf(-fabsf(raw))));
    float s = __fmul_rn(s0, sp);
    return (s > smax) ? smax : s;
}

// ------------------------------------------------------------------------
// Generic kernel
// ------------------------------------------------------------------------
template <typename T, bool MS>
__global__ void __launch_bounds__(256)
fwd_generic_kernel(Geometry g, const T *__restrict__ in, const T *__restrict__ ow,
                   T *__restrict__ out, const __grid_constant__ MsdcnParams ms) {
    constexpr int CH = 8;
    const int nch = (g.D + CH - 1) / CH;
    const long long total = (long long)g.N * g.Ho * g.Wo * g.G * nch;
    const size_t img = (size_t)g.H * g.W * g.C;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (long long)gridDim.x * blockDim.x) {
        const int ch = (int)(t % nch);
        const long long r = t / nch;
        const int grp = (int)(r % g.G);
        const long long pix = r / g.G;
        const int wo = (int)(pix % g.Wo);
        const long long r2 = pix / g.Wo;
        const int ho = (int)(r2 % g.Ho);
        const int n = (int)(r2 / g.Ho);
        const int d0 = ch * CH;
        const int cnt = min(CH, g.D - d0);
        const T *rec = ow + (size_t)(pix * g.G + grp) * g.K * 3;
        float s = 1.0f;
        if (MS) {
            const float raw = Elem<T>::to_f(static_cast<const T *>(ms.raw)[pix * g.G + grp]);
            s = msdcn_scale(raw, ms.s0[grp], ms.smax);
        }
        float acc[CH];
#pragma unroll
        for (int d = 0; d < CH; ++d) acc[d] = 0.0f;
        const T *src = in + (size_t)n * img + (size_t)grp * g.D + d0;
        for (int i = 0; i < g.kh; ++i) {
            for (int j = 0; j < g.kw; ++j) {
                const int k = i * g.kw + j;
                float dx = Elem<T>::to_f(rec[3 * k]);
                float dy = Elem<T>::to_f(rec[3 * k + 1]);
                const float m = Elem<T>::to_f(rec[3 * k + 2]);
                if (MS) {
                    dx = __fmul_rn(s, dx);
                    dy = __fmul_rn(s, dy);
                }
                const float x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                const float y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
                if (!(x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H)) continue;
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const int x0 = (int)x0f, y0 = (int)y0f;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int yy = y0 + a, xx = x0 + b;
                        if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                        const float w = (a ? ly : 1.0f - ly) * (b ? lx : 1.0f - lx) * m;
                        const T *p = src + ((size_t)yy * g.W + xx) * g.C;
#pragma unroll
                        for (int d = 0; d < CH; ++d)
                            if (d < cnt) acc[d] = fmaf(w, Elem<T>::to_f(p[d]), acc[d]);
                    }
                }
            }
        }
        T *dst = out + (size_t)pix * g.C + (size_t)grp * g.D + d0;
#pragma unroll
        for (int d = 0; d < CH; ++d)
            if (d < cnt) dst[d] = Elem<T>::from_f(acc[d]);
    }
}

// ------------------------------------------------------------------------
// Shared-memory halo kernel (3x3 taps, D*sizeof(T) = 16*U bytes)
// ------------------------------------------------------------------------

// Shared-memory byte layout of one halo CTA.
struct HaloSmem {
    static __host__ __device__ __forceinline__ int slots_offset(const HaloPlan &p) {
        return p.halo_bytes;
    }
    static __host__ __device__ __forceinline__ int barrier_offset(const HaloPlan &p) {
        return p.halo_bytes + p.TH * p.TW * p.slot_bytes;
    }
};

// Reads the 27 (dx, dy, m) values of one record from shared memory.
template <typename T> struct RecordReader;
template <> struct RecordReader<float> {
    static __device__ __forceinline__ void read(const unsigned char *rec, float (&v)[27]) {
        const float *p = reinterpret_cast<const float *>(rec);
#pragma unroll
        for (int i = 0; i < 27; ++i) v[i] = p[i];
    }
};
template <typename T16> struct RecordReader16 {
    // The record starts on a 2-byte boundary: read 15 aligned words and shift
    // by half a word when the record starts mid-word.
    static __device__ __forceinline__ void read(const unsigned char *rec, float (&v)[27]) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(rec);
        const unsigned *w = reinterpret_cast<const unsigned *>(a & ~uintptr_t(3));
        const unsigned sh = (unsigned)(a & 2u) * 8u;  // 0 or 16 bits
        unsigned wd[15];
#pragma unroll
        for (int i = 0; i < 15; ++i) wd[i] = w[i];
#pragma unroll
        for (int i = 0; i < 14; ++i) {
            const unsigned u = __funnelshift_r(wd[i], wd[i + 1], sh);
            v[2 * i] = cvt_lo(u);
            if (2 * i + 1 < 27) v[2 * i + 1] = cvt_hi(u);
        }
    }
    static __device__ __forceinline__ float cvt_lo(unsigned u);
    static __device__ __forceinline__ float cvt_hi(unsigned u);
};
template <> __device__ __forceinline__ float RecordReader16<__nv_bfloat16>::cvt_lo(unsigned u) {
    return __uint_as_float(u << 16);
}
template <> __device__ __forceinline__ float RecordReader16<__nv_bfloat16>::cvt_hi(unsigned u) {
    return __uint_as_float(u & 0xffff0000u);
}
template <> __device__ __forceinline__ float RecordReader16<__half>::cvt_lo(unsigned u) {
    return __half2float(__ushort_as_half((unsigned short)(u & 0xffffu)));
}
template <> __device__ __forceinline__ float RecordReader16<__half>::cvt_hi(unsigned u) {
    return __half2float(__ushort_as_half((unsigned short)(u >> 16)));
}
template <> struct RecordReader<__nv_bfloat16> : RecordReader16<__nv_bfloat16> {};
template <> struct RecordReader<__half> : RecordReader16<__half> {};

// Reads tap k's (dx, dy, m) of a record in shared memory (escape path).
template <typename T>
__device__ __forceinline__ void record_tap(const unsigned char *rec, int k, float &dx, float &dy,
                                           float &m) {
    const T *p = reinterpret_cast<const T *>(rec) + 3 * k;
    dx = Elem<T>::to_f(p[0]);
    dy = Elem<T>::to_f(p[1]);
    m = Elem<T>::to_f(p[2]);
}

template <typename T, int U, bool MS, bool OS1, bool MIXED>
__global__ void __launch_bounds__(256, (U >= 8 ? 1 : 2))
fwd_halo_kernel(const __grid_constant__ CUtensorMap tmap, Geometry g, HaloPlan pl,
                const T *__restrict__ in, const T *__restrict__ ow, T *__restrict__ out,
                unsigned long long ow_bytes, const __grid_constant__ MsdcnParams ms) {
    constexpr int EB = Elem<T>::kBytes;
    constexpr int VE = Elem<T>::kPerVec;  // elements per 16-byte chunk
    constexpr int REC = 27 * EB;          // bytes of one (pixel, group) record
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *halo = smem;
    unsigned char *slots = smem + HaloSmem::slots_offset(pl);
    const uint32_t bar = smem_u32(smem + HaloSmem::barrier_offset(pl));

    // ---- which tile ----
    int b = blockIdx.x;
    const int tw = b % pl.tiles_w;
    b /= pl.tiles_w;
    const int th = b % pl.tiles_h;
    b /= pl.tiles_h;
    const int sl = b % pl.slices;
    const int n = b / pl.slices;
    const int ho0 = th * pl.TH, wo0 = tw * pl.TW, g0 = sl * pl.Gc;
    const int hy0 = pl.full_h ? -1 : ho0 * g.sh - g.ph - pl.R;
    const int hx0 = pl.full_w ? -1 : wo0 * g.sw - g.pw - pl.R;
    const int th_eff = min(pl.TH, g.Ho - ho0), tw_eff = min(pl.TW, g.Wo - wo0);
    const int D = g.D;
    const int PS = pl.Gc * D * EB;  // bytes per halo pixel
    const int RS = pl.HC * PS;      // bytes per halo row

    if (threadIdx.x == 0) {
        mbar_init(bar, blockDim.x);
        fence_barrier_init();
    }
    __syncthreads();

    // ---- stage: halo (thread 0) + one record slot per tile pixel ----
    {
        uint32_t tx_bytes = 0;
        if (threadIdx.x == 0) tx_bytes = (uint32_t)pl.HR * pl.HC * PS;
        const int npix = pl.TH * pl.TW;
        for (int p = threadIdx.x; p < npix; p += blockDim.x) {
            const int ty = p / pl.TW, tx = p - ty * pl.TW;
            if (ty >= th_eff || tx >= tw_eff) continue;
            const unsigned long long gp = ((unsigned long long)n * g.Ho + ho0 + ty) * g.Wo + wo0 + tx;
            const unsigned long long start = (gp * g.G + g0) * (unsigned long long)REC;
            const unsigned long long end = start + (unsigned long long)pl.Gc * REC;
            const unsigned long long a = start & ~15ull;
            const unsigned long long e = min((end + 15ull) & ~15ull, ow_bytes & ~15ull);
            if (e > a) tx_bytes += (uint32_t)(e - a);
        }
        mbar_arrive_expect_tx(bar, tx_bytes);
        if (threadIdx.x == 0)
            tma_load_4d(smem_u32(halo), &tmap, g0 * D, hx0, hy0, n, bar);
        for (int p = threadIdx.x; p < npix; p += blockDim.x) {
            const int ty = p / pl.TW, tx = p - ty * pl.TW;
            if (ty >= th_eff || tx >= tw_eff) continue;
            const unsigned long long gp = ((unsigned long long)n * g.Ho + ho0 + ty) * g.Wo + wo0 + tx;
            const unsigned long long start = (gp * g.G + g0) * (unsigned long long)REC;
            const unsigned long long end = start + (unsigned long long)pl.Gc * REC;
            const unsigned long long a = start & ~15ull;
            const unsigned long long e = min((end + 15ull) & ~15ull, ow_bytes & ~15ull);
            unsigned char *slot = slots + (size_t)p * pl.slot_bytes;
            if (e > a)
                bulk_load(smem_u32(slot), reinterpret_cast<const unsigned char *>(ow) + a,
                          (uint32_t)(e - a), bar);
            // the tensor's last bytes when its size is not a multiple of 16
            for (unsigned long long q = e; q < end; q += EB) {
                const unsigned char *sp = reinterpret_cast<const unsigned char *>(ow) + q;
                if (EB == 4)
                    *reinterpret_cast<unsigned *>(slot + (q - a)) = *reinterpret_cast<const unsigned *>(sp);
                else
                    *reinterpret_cast<unsigned short *>(slot + (q - a)) =
                        *reinterpret_cast<const unsigned short *>(sp);
            }
        }
    }
    const bool ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
        if (threadIdx.x == 0) atomicOr(&g_error_word, kErrTimeout);
        mbar_wait_bounded(bar, 0, kWaitLimitNs);  // let copies in flight land
        return;
    }

    // ---- one thread per (pixel, group) ----
    const int lane = threadIdx.x & 31;
    const int npairs = pl.TH * pl.TW * pl.Gc;
    const size_t img = (size_t)g.H * g.W * g.C;
    // the staged window in image coordinates: corners x0, x0+1 are inside iff
    // hx_lo <= x < hx_hi (NaN fails the test and goes to the escape path)
    const float hx_lo = (float)hx0, hx_hi = (float)(hx0 + pl.HC - 1);
    const float hy_lo = (float)hy0, hy_hi = (float)(hy0 + pl.HR - 1);
    const float PSf = (float)PS, RSf = (float)RS;
    const float dwf = (float)g.dw, dhf = (float)g.dh;
    for (int f = threadIdx.x; f < npairs; f += blockDim.x) {
        const int pix = f / pl.Gc;
        const int gl = f - pix * pl.Gc;
        const int ty = pix / pl.TW, tx = pix - ty * pl.TW;
        if (ty >= th_eff || tx >= tw_eff) continue;
        const int ho = ho0 + ty, wo = wo0 + tx;
        const unsigned long long gp = ((unsigned long long)n * g.Ho + ho) * g.Wo + wo;
        const unsigned long long start = (gp * g.G + g0) * (unsigned long long)REC;
        const unsigned char *rec = slots + (size_t)pix * pl.slot_bytes + (start & 15ull) + gl * REC;
        float v[27];
        RecordReader<T>::read(rec, v);
        float s = 1.0f;
        if (MS) {
            const float raw = Elem<T>::to_f(static_cast<const T *>(ms.raw)[gp * g.G + g0 + gl]);
            s = msdcn_scale(raw, ms.s0[g0 + gl], ms.smax);
#pragma unroll
            for (int k = 0; k < 9; ++k) {
                v[3 * k] = __fmul_rn(s, v[3 * k]);
                v[3 * k + 1] = __fmul_rn(s, v[3 * k + 1]);
            }
        }
        // chunk rotation: lanes of one 8-lane phase start at different chunks
        const int r = (U <= 8) ? (((lane & 7) * U) >> 3) : (f & (U - 1));
        float acc[U][VE];
#pragma unroll
        for (int c = 0; c < U; ++c)
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[c][e] = 0.0f;

        const float fbx = (float)(wo * g.sw - g.pw), fby = (float)(ho * g.sh - g.ph);
        const float bxs[3] = {fbx, fbx + dwf, fbx + 2.0f * dwf};
        const float bys[3] = {fby, fby + dhf, fby + 2.0f * dhf};
        const unsigned char *hbase = halo + (size_t)gl * D * EB;
        unsigned esc = 0;
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            const float x = OS1 ? __fadd_rn(bxs[k % 3], v[3 * k])
                                : __fadd_rn(bxs[k % 3], __fmul_rn(v[3 * k], g.os));
            const float y = OS1 ? __fadd_rn(bys[k / 3], v[3 * k + 1])
                                : __fadd_rn(bys[k / 3], __fmul_rn(v[3 * k + 1], g.os));
            const float m = v[3 * k + 2];
            if (x >= hx_lo && x < hx_hi && y >= hy_lo && y < hy_hi) {
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const float mly = m * ly, mhy = m - mly;
                const float w01 = mhy * lx, w00 = mhy - w01;
                const float w11 = mly * lx, w10 = mly - w11;
                // integer-valued floats below 2^24: the byte offset is exact
                const int off = __float2int_rz(fmaf(y0f - hy_lo, RSf, (x0f - hx_lo) * PSf));
                const unsigned char *c00 = hbase + off;
#pragma unroll
                for (int c = 0; c < U; ++c) {
                    const int o = ((c + r) & (U - 1)) * 16;
                    const uint4 q00 = *reinterpret_cast<const uint4 *>(c00 + o);
                    const uint4 q01 = *reinterpret_cast<const uint4 *>(c00 + PS + o);
                    const uint4 q10 = *reinterpret_cast<const uint4 *>(c00 + RS + o);
                    const uint4 q11 = *reinterpret_cast<const uint4 *>(c00 + RS + PS + o);
                    if (MIXED) {
                        VecMathMixed<T>::fma(acc[c], q00, w00);
                        VecMathMixed<T>::fma(acc[c], q01, w01);
                        VecMathMixed<T>::fma(acc[c], q10, w10);
                        VecMathMixed<T>::fma(acc[c], q11, w11);
                    } else {
                        VecMath<T>::fma(acc[c], q00, w00);
                        VecMath<T>::fma(acc[c], q01, w01);
                        VecMath<T>::fma(acc[c], q10, w10);
                        VecMath<T>::fma(acc[c], q11, w11);
                    }
                }
            } else {
                esc |= 1u << k;
            }
        }
        // samples outside the staged window (rare): 16-byte loads from global
        // memory, each corner tested against the image
        const T *gbase = in + (size_t)n * img + (size_t)(g0 + gl) * D;
        while (esc) {
            const int k = __ffs(esc) - 1;
            esc &= esc - 1;
            float dx, dy, m;
            record_tap<T>(rec, k, dx, dy, m);
            if (MS) {
                dx = __fmul_rn(s, dx);
                dy = __fmul_rn(s, dy);
            }
            const int i = k / 3, j = k - 3 * (k / 3);
            const float x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
            const float y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
            if (!(x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H)) continue;
            const float x0f = floorf(x), y0f = floorf(y);
            const float lx = x - x0f, ly = y - y0f;
            const float mly = m * ly, mhy = m - mly;
            const float w01 = mhy * lx, w11 = mly * lx;
            const float wc[4] = {mhy - w01, w01, mly - w11, w11};
            const int x0 = (int)x0f, y0 = (int)y0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int yy = y0 + (q >> 1), xx = x0 + (q & 1);
                if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                const uint4 *p = reinterpret_cast<const uint4 *>(gbase + ((size_t)yy * g.W + xx) * g.C);
#pragma unroll
                for (int c = 0; c < U; ++c)
                    VecMath<T>::fma(acc[c], __ldg(p + ((c + r) & (U - 1))), wc[q]);
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + gp * g.C + (size_t)(g0 + gl) * D);
#pragma unroll
        for (int c = 0; c < U; ++c) dst[(c + r) & (U - 1)] = VecMath<T>::pack(acc[c]);
    }
}

}  // namespace dcn4
