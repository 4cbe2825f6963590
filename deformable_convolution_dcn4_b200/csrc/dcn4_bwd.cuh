// dcn4_bwd.cuh -- backward kernels of DCNv4 deformable spatial aggregation.
//
// The forward is out[p0, g*D+d] = sum_k m_k * sum_corners w_c(lx, ly) *
// in[corner, g*D+d] (DCNv4 digest "方法1. 消除冗余工作负载"; FlowDCN "2.2"), so with
// go = grad_out[p0, g*D + .] and V_c the corner vectors:
//   d/dm_k   = sum_c w_c <go, V_c>
//   d/ddx_k  = offset_scale * m_k * sum_c (dw_c/dlx) <go, V_c>,  dw/dlx = +-wy
//   d/ddy_k  = offset_scale * m_k * sum_c (dw_c/dly) <go, V_c>,  dw/dly = +-wx
//   grad_in[corner c] += m_k * w_c * go
// grad_in is gathered from many output pixels, so it accumulates in fp32
// with atomic adds into a zeroed buffer, converted to the element type last.
#pragma once

#include "dcn4_common.cuh"

namespace dcn4 {

// One thread per (pixel, group); scalar loads; any shape and alignment.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_generic_kernel(Geometry g, const T *__restrict__ in, const T *__restrict__ ow,
                   const T *__restrict__ gout, float *__restrict__ gin, T *__restrict__ gow) {
    const long long total = (long long)g.N * g.Ho * g.Wo * g.G;
    const size_t img = (size_t)g.H * g.W * g.C;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (long long)gridDim.x * blockDim.x) {
        const int grp = (int)(t % g.G);
        const long long pix = t / g.G;
        const int wo = (int)(pix % g.Wo);
        const long long r2 = pix / g.Wo;
        const int ho = (int)(r2 % g.Ho);
        const int n = (int)(r2 / g.Ho);
        const T *rec = ow + (size_t)t * g.K * 3;
        T *grec = gow + (size_t)t * g.K * 3;
        const T *go = gout + (size_t)pix * g.C + (size_t)grp * g.D;
        const T *src = in + (size_t)n * img + (size_t)grp * g.D;
        float *dst = gin + (size_t)n * img + (size_t)grp * g.D;
        for (int i = 0; i < g.kh; ++i) {
            for (int j = 0; j < g.kw; ++j) {
                const int k = i * g.kw + j;
                const float dx = Elem<T>::to_f(rec[3 * k]);
                const float dy = Elem<T>::to_f(rec[3 * k + 1]);
                const float m = Elem<T>::to_f(rec[3 * k + 2]);
                const float x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                const float y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
                float gx = 0.0f, gy = 0.0f, gm = 0.0f;
                if (x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H) {
                    const float x0f = floorf(x), y0f = floorf(y);
                    const float lx = x - x0f, ly = y - y0f;
                    const int x0 = (int)x0f, y0 = (int)y0f;
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
#pragma unroll
                        for (int b = 0; b < 2; ++b) {
                            const int yy = y0 + a, xx = x0 + b;
                            if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                            const float wy = a ? ly : 1.0f - ly;
                            const float wx = b ? lx : 1.0f - lx;
                            const float w = wy * wx;
                            const size_t at = ((size_t)yy * g.W + xx) * g.C;
                            float dot = 0.0f;
                            for (int d = 0; d < g.D; ++d) {
                                const float god = Elem<T>::to_f(go[d]);
                                dot = fmaf(god, Elem<T>::to_f(src[at + d]), dot);
                                atomicAdd(dst + at + d, m * w * god);
                            }
                            gm = fmaf(w, dot, gm);
                            gx = fmaf(b ? wy : -wy, dot, gx);
                            gy = fmaf(a ? wx : -wx, dot, gy);
                        }
                    }
                }
                grec[3 * k] = Elem<T>::from_f(g.os * m * gx);
                grec[3 * k + 1] = Elem<T>::from_f(g.os * m * gy);
                grec[3 * k + 2] = Elem<T>::from_f(gm);
            }
        }
    }
}

// Zeroes `n` floats (16-byte vector body + scalar tail).
__global__ void __launch_bounds__(256) zero_f32_kernel(float *__restrict__ p, long long n) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long nv = ((reinterpret_cast<uintptr_t>(p) & 15) == 0) ? n / 4 : 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride)
        reinterpret_cast<float4 *>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long i = nv * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        p[i] = 0.0f;
}

// Zeroes `bytes` bytes (16-byte vector body when aligned, byte tail).
__global__ void __launch_bounds__(256) zero_bytes_kernel(unsigned char *__restrict__ p, long long bytes) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long nv = ((reinterpret_cast<uintptr_t>(p) & 15) == 0) ? bytes / 16 : 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride)
        reinterpret_cast<uint4 *>(p)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (long long i = nv * 16 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < bytes; i += stride)
        p[i] = 0;
}

// dst[i] = T(src[i]) for n elements, rounding to nearest.
template <typename T>
__global__ void __launch_bounds__(256)
convert_f32_kernel(const float *__restrict__ src, T *__restrict__ dst, long long n) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) && sizeof(T) == 2;
    const long long nv = vec ? n / 4 : 0;
    if constexpr (sizeof(T) == 2) {
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
            const float4 f = reinterpret_cast<const float4 *>(src)[i];
            uint2 o;
            o.x = VecMath<T>::pk(f.x, f.y);
            o.y = VecMath<T>::pk(f.z, f.w);
            reinterpret_cast<uint2 *>(dst)[i] = o;
        }
    }
    for (long long i = nv * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        dst[i] = Elem<T>::from_f(src[i]);
}

}  // namespace dcn4
