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
// MS: the FlowDCN multi-scale variant ("3.1"): ow holds (dir_x, dir_y, m),
// the offset is s * dir with s = msdcn_scale(raw); by the chain rule
// d/d dir = s * d/d offset and d/d raw = (ds/draw) * sum_k <d/d offset_k, dir_k>,
// written to graw [N][Ho][Wo][G].
template <typename T, bool MS>
__global__ void __launch_bounds__(256)
bwd_generic_kernel(Geometry g, const T *__restrict__ in, const T *__restrict__ ow,
                   const T *__restrict__ gout, float *__restrict__ gin, T *__restrict__ gow,
                   const __grid_constant__ MsdcnParams ms, T *__restrict__ graw) {
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
        const unsigned long long owb = ow_bytes_of(g, sizeof(T));
        if (!DCN4_GMEM_OK(rec, g.K * 3 * sizeof(T), ow, owb) ||
            !DCN4_GMEM_OK(grec, g.K * 3 * sizeof(T), gow, owb) ||
            !DCN4_GMEM_OK(go, g.D * sizeof(T), gout, output_bytes(g, sizeof(T))) ||
            (MS && !DCN4_GMEM_OK(static_cast<const T *>(ms.raw) + t, sizeof(T), ms.raw,
                                 raw_bytes(g, sizeof(T)))) ||
            (MS && !DCN4_GMEM_OK(graw + t, sizeof(T), graw, raw_bytes(g, sizeof(T)))))
            continue;
        float s = 1.0f, gs = 0.0f;
        if (MS) s = msdcn_scale(Elem<T>::to_f(static_cast<const T *>(ms.raw)[t]), ms.s0[grp], ms.smax);
        // DCNv3 weights: softmax over the taps; the gradients with respect to
        // the weights are kept (fp32, up to kMaxTaps) to form the logit
        // gradient w_k (gw_k - sum_j w_j gw_j) after the loop
        SoftmaxNorm sn{0.0f, 1.0f};
        float gwk[kMaxTaps];
        float dotw = 0.0f;
        if (!MS && g.softmax) {
            float mx = -INFINITY, sum = 0.0f;
            for (int k = 0; k < g.K; ++k) mx = fmaxf(mx, Elem<T>::to_f(rec[3 * k + 2]));
            for (int k = 0; k < g.K; ++k) sum += expf(Elem<T>::to_f(rec[3 * k + 2]) - mx);
            sn = SoftmaxNorm{mx, 1.0f / sum};
        }
        for (int i = 0; i < g.kh; ++i) {
            for (int j = 0; j < g.kw; ++j) {
                const int k = i * g.kw + j;
                const float dx = Elem<T>::to_f(rec[3 * k]);
                const float dy = Elem<T>::to_f(rec[3 * k + 1]);
                float m = Elem<T>::to_f(rec[3 * k + 2]);
                if (!MS && g.softmax) m = sn.weight(m);
                float x, y, dsx = 0.0f, dsy = 0.0f;  // ds*: d position / d s (MSDCN)
                if (MS) {
                    x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, j, g.kw, g.dw, s, dx, g.os, &dsx);
                    y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, i, g.kh, g.dh, s, dy, g.os, &dsy);
                } else {
                    x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                    y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
                }
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
                            if (!DCN4_GMEM_OK(src + at, g.D * sizeof(T), in, input_bytes(g, sizeof(T))) ||
                                !DCN4_GMEM_OK(dst + at, g.D * 4, gin, input_bytes(g, 4)))
                                continue;
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
                const float tx = g.os * m * gx, ty = g.os * m * gy;  // d/d offset
                grec[3 * k] = Elem<T>::from_f(MS && tx != 0.0f ? s * tx : tx);
                grec[3 * k + 1] = Elem<T>::from_f(MS && ty != 0.0f ? s * ty : ty);
                if (!MS && g.softmax) {
                    gwk[k] = gm;
                    dotw = fmaf(m, gm, dotw);
                } else {
                    grec[3 * k + 2] = Elem<T>::from_f(gm);
                }
                if (MS) gs = fmaf(m * gx, dsx, fmaf(m * gy, dsy, gs));
            }
        }
        if (!MS && g.softmax)
            for (int k = 0; k < g.K; ++k)
                grec[3 * k + 2] = Elem<T>::from_f(
                    sn.weight(Elem<T>::to_f(rec[3 * k + 2])) * (gwk[k] - dotw));
        if (MS) {
            const float raw = Elem<T>::to_f(static_cast<const T *>(ms.raw)[t]);
            graw[t] = Elem<T>::from_f(gs == 0.0f ? 0.0f : gs * msdcn_scale_grad(raw, ms.s0[grp], ms.smax));
        }
    }
}

// Zeroes `n` floats (16-byte vector body + scalar tail).
__global__ void __launch_bounds__(256) zero_f32_kernel(float *__restrict__ p, long long n) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long nv = ((reinterpret_cast<uintptr_t>(p) & 15) == 0) ? n / 4 : 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride)
        if (DCN4_CHECK(4 * i + 4 <= n)) reinterpret_cast<float4 *>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long i = nv * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        p[i] = 0.0f;
}

// Zeroes `bytes` bytes (16-byte vector body when aligned, byte tail).
__global__ void __launch_bounds__(256) zero_bytes_kernel(unsigned char *__restrict__ p, long long bytes) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long nv = ((reinterpret_cast<uintptr_t>(p) & 15) == 0) ? bytes / 16 : 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride)
        if (DCN4_CHECK(16 * i + 16 <= bytes)) reinterpret_cast<uint4 *>(p)[i] = make_uint4(0u, 0u, 0u, 0u);
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
            if (!DCN4_CHECK(4 * i + 4 <= n)) continue;
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
