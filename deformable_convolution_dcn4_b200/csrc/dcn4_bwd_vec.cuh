// dcn4_bwd_vec.cuh -- vectorised global-memory forward and backward of DCNv4
// and of the FlowDCN multi-scale variant, for the calls the shared-memory
// kernels do not take (MSDCN backward, group widths other than 32-128 bytes,
// kernel sizes other than 3x3).
// Included after dcn4_bwd_halo.cuh (uses its DotF, ChunkUnpack, red_add_v4).
//
// LPP = D * sizeof(T) / 16 lanes share one (pixel, group): lane `sub` owns
// channels [sub*VE, sub*VE + VE) of the group (one 16-byte vector). Per tap
// every lane loads its 16 bytes of each in-image corner, forms its share of
// the four dot products <grad_out, V_c>, and the shares are summed across the
// LPP lanes with xor shuffles; every lane then knows the three gradients of
// the tap and adds m * w_c * grad_out for its channels to the fp32 workspace
// with 16-byte vector atomics. The derivatives are those of bwd_generic_kernel
// (dcn4_bwd.cuh), including the MSDCN chain rule and the DCNv3 softmax.
#pragma once

#include "dcn4_bwd_halo.cuh"

namespace dcn4 {

// Forward: thread t of a (pixel, group)'s VPP = D*sizeof(T)/16 threads owns
// one 16-byte vector of the group's channels; per tap it loads that vector
// of each in-image corner (L1/L2) and accumulates in fp32. Positions,
// weights and the MSDCN scale / DCNv3 softmax are formed as in
// fwd_generic_kernel (dcn4_fwd.cuh); no lane exchanges anything.
template <typename T, bool MS>
__global__ void __launch_bounds__(256)
fwd_vec_kernel(Geometry g, const T *__restrict__ in, const T *__restrict__ ow,
               T *__restrict__ out, const __grid_constant__ MsdcnParams ms) {
    constexpr int VE = Elem<T>::kPerVec;
    const int vpp = g.D / VE;
    const long long total = (long long)g.N * g.Ho * g.Wo * g.G * vpp;
    const size_t img = (size_t)g.H * g.W * g.C;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (long long)gridDim.x * blockDim.x) {
        const int sub = (int)(t % vpp);
        const long long pr = t / vpp;
        const int grp = (int)(pr % g.G);
        const long long pix = pr / g.G;
        const int wo = (int)(pix % g.Wo);
        const long long r2 = pix / g.Wo;
        const int ho = (int)(r2 % g.Ho);
        const int n = (int)(r2 / g.Ho);
        const T *rec = ow + (size_t)pr * g.K * 3;
        const int c0 = grp * g.D + sub * VE;
        const T *src = in + (size_t)n * img + c0;
        if (!DCN4_GMEM_OK(rec, g.K * 3 * sizeof(T), ow, ow_bytes_of(g, sizeof(T))) ||
            !DCN4_GMEM_OK(out + (size_t)pix * g.C + c0, 16, out, output_bytes(g, sizeof(T))) ||
            (MS && !DCN4_GMEM_OK(static_cast<const T *>(ms.raw) + pr, sizeof(T), ms.raw,
                                 raw_bytes(g, sizeof(T)))))
            continue;
        float s = 1.0f;
        if (MS) s = msdcn_scale(Elem<T>::to_f(static_cast<const T *>(ms.raw)[pr]), ms.s0[grp], ms.smax);
        SoftmaxNorm sn{0.0f, 1.0f};
        if (!MS && g.softmax) {
            float mx = -INFINITY, sum = 0.0f;
            for (int k = 0; k < g.K; ++k) mx = fmaxf(mx, Elem<T>::to_f(rec[3 * k + 2]));
            for (int k = 0; k < g.K; ++k) sum += expf(Elem<T>::to_f(rec[3 * k + 2]) - mx);
            sn = SoftmaxNorm{mx, 1.0f / sum};
        }
        float acc[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] = 0.0f;
        for (int i = 0; i < g.kh; ++i) {
            for (int j = 0; j < g.kw; ++j) {
                const int k = i * g.kw + j;
                const float dx = Elem<T>::to_f(rec[3 * k]);
                const float dy = Elem<T>::to_f(rec[3 * k + 1]);
                float m = Elem<T>::to_f(rec[3 * k + 2]);
                if (!MS && g.softmax) m = sn.weight(m);
                float x, y, dsx, dsy;
                if (MS) {
                    x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, j, g.kw, g.dw, s, dx, g.os, &dsx);
                    y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, i, g.kh, g.dh, s, dy, g.os, &dsy);
                } else {
                    x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                    y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
                }
                if (!(x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H)) continue;
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const int x0 = (int)x0f, y0 = (int)y0f;
                uint4 q[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int yy = y0 + (c >> 1), xx = x0 + (c & 1);
                    q[c] = (yy >= 0 && yy < g.H && xx >= 0 && xx < g.W)
                               ? DCN4_LDG16(src + ((size_t)yy * g.W + xx) * g.C, in,
                                            input_bytes(g, sizeof(T)))
                               : make_uint4(0u, 0u, 0u, 0u);
                }
                const float mly = m * ly, mhy = m - mly;
                VecMath<T>::fma(acc, q[0], mhy - mhy * lx);
                VecMath<T>::fma(acc, q[1], mhy * lx);
                VecMath<T>::fma(acc, q[2], mly - mly * lx);
                VecMath<T>::fma(acc, q[3], mly * lx);
            }
        }
        *reinterpret_cast<uint4 *>(out + (size_t)pix * g.C + c0) = VecMath<T>::pack(acc);
    }
}

template <typename T, bool MS, int LPP>
__global__ void __launch_bounds__(256)
bwd_vec_kernel(Geometry g, const T *__restrict__ in, const T *__restrict__ ow,
               const T *__restrict__ gout, float *__restrict__ gin, T *__restrict__ gow,
               const __grid_constant__ MsdcnParams ms, T *__restrict__ graw) {
    constexpr int VE = Elem<T>::kPerVec;
    const long long pairs = (long long)g.N * g.Ho * g.Wo * g.G;
    const long long total = pairs * LPP;
    const size_t img = (size_t)g.H * g.W * g.C;
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // the loop runs in whole warps so that every shuffle has all 32 lanes
    for (long long base = (long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total;
         base += stride) {
        const long long t = base + lane;
        const bool active = t < total;
        const long long pr = active ? t / LPP : 0;
        const int sub = (int)(t % LPP);
        const int grp = (int)(pr % g.G);
        const long long pix = pr / g.G;
        const int wo = (int)(pix % g.Wo);
        const long long r2 = pix / g.Wo;
        const int ho = (int)(r2 % g.Ho);
        const int n = (int)(r2 / g.Ho);
        const T *rec = ow + (size_t)pr * g.K * 3;
        T *grec = gow + (size_t)pr * g.K * 3;
        const int c0 = grp * g.D + sub * VE;  // this lane's first channel
        const unsigned long long owb = ow_bytes_of(g, sizeof(T)), rawb = raw_bytes(g, sizeof(T));
        const bool in_range =
            !active || (DCN4_GMEM_OK(rec, g.K * 3 * sizeof(T), ow, owb) &&
                        DCN4_GMEM_OK(grec, g.K * 3 * sizeof(T), gow, owb) &&
                        (!MS || (DCN4_GMEM_OK(static_cast<const T *>(ms.raw) + pr, sizeof(T), ms.raw,
                                              rawb) &&
                                 DCN4_GMEM_OK(graw + pr, sizeof(T), graw, rawb))));
        // a lane whose tensors fail the checked build's bounds takes no part
        // (it still runs the shuffles, as an inactive lane)
        const bool act = active && in_range;
        float gof[VE];
        ChunkUnpack<T>::get(act ? DCN4_LDG16(gout + (size_t)pix * g.C + c0, gout,
                                             output_bytes(g, sizeof(T)))
                                : make_uint4(0u, 0u, 0u, 0u),
                            gof);
        const T *src = in + (size_t)n * img + c0;
        float *dst = gin + (size_t)n * img + c0;
        float s = 1.0f, gs = 0.0f;
        if (MS && act)
            s = msdcn_scale(Elem<T>::to_f(static_cast<const T *>(ms.raw)[pr]), ms.s0[grp], ms.smax);
        SoftmaxNorm sn{0.0f, 1.0f};
        if (!MS && g.softmax && act) {
            float mx = -INFINITY, sum = 0.0f;
            for (int k = 0; k < g.K; ++k) mx = fmaxf(mx, Elem<T>::to_f(rec[3 * k + 2]));
            for (int k = 0; k < g.K; ++k) sum += expf(Elem<T>::to_f(rec[3 * k + 2]) - mx);
            sn = SoftmaxNorm{mx, 1.0f / sum};
        }
        float dotw = 0.0f;  // sum_k w_k * d/dw_k (softmax)
        for (int i = 0; i < g.kh; ++i) {
            for (int j = 0; j < g.kw; ++j) {
                const int k = i * g.kw + j;
                float dx = 0.0f, dy = 0.0f, m = 0.0f;
                if (act) {
                    dx = Elem<T>::to_f(rec[3 * k]);
                    dy = Elem<T>::to_f(rec[3 * k + 1]);
                    m = Elem<T>::to_f(rec[3 * k + 2]);
                }
                if (!MS && g.softmax) m = sn.weight(m);
                float x, y, dsx = 0.0f, dsy = 0.0f;
                if (MS) {
                    x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, j, g.kw, g.dw, s, dx, g.os, &dsx);
                    y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, i, g.kh, g.dh, s, dy, g.os, &dsy);
                } else {
                    x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                    y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
                }
                const bool inside =
                    act && x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H;
                float lx = 0.0f, ly = 0.0f;
                int x0 = 0, y0 = 0;
                float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                if (inside) {
                    const float x0f = floorf(x), y0f = floorf(y);
                    lx = x - x0f;
                    ly = y - y0f;
                    x0 = (int)x0f;
                    y0 = (int)y0f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int yy = y0 + (q >> 1), xx = x0 + (q & 1);
                        if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                        d[q] = DotF<T>::dot(DCN4_LDG16(src + ((size_t)yy * g.W + xx) * g.C, in,
                                                       input_bytes(g, sizeof(T))),
                                            gof);
                    }
                }
#pragma unroll
                for (int o = LPP / 2; o > 0; o >>= 1)
#pragma unroll
                    for (int q = 0; q < 4; ++q) d[q] += __shfl_xor_sync(0xffffffffu, d[q], o);
                float gx = 0.0f, gy = 0.0f, gm = 0.0f;
                if (inside) {
                    const float hx = 1.0f - lx, hy = 1.0f - ly;
                    gm = hy * (hx * d[0] + lx * d[1]) + ly * (hx * d[2] + lx * d[3]);
                    gx = hy * (d[1] - d[0]) + ly * (d[3] - d[2]);
                    gy = hx * (d[2] - d[0]) + lx * (d[3] - d[1]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int yy = y0 + (q >> 1), xx = x0 + (q & 1);
                        if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                        const float w = m * ((q >> 1) ? ly : hy) * ((q & 1) ? lx : hx);
                        float *p = dst + ((size_t)yy * g.W + xx) * g.C;
                        if (!DCN4_GMEM_OK(p, VE * 4, gin, input_bytes(g, 4))) continue;
#pragma unroll
                        for (int e = 0; e < VE; e += 4)
                            red_add_v4(p + e, w * gof[e], w * gof[e + 1], w * gof[e + 2],
                                       w * gof[e + 3]);
                    }
                }
                const float tx = g.os * m * gx, ty = g.os * m * gy;  // d/d offset
                if (act && sub == 0) {
                    grec[3 * k] = Elem<T>::from_f(MS && tx != 0.0f ? s * tx : tx);
                    grec[3 * k + 1] = Elem<T>::from_f(MS && ty != 0.0f ? s * ty : ty);
                    grec[3 * k + 2] = Elem<T>::from_f(gm);
                }
                dotw = fmaf(m, gm, dotw);
                if (MS) gs = fmaf(m * gx, dsx, fmaf(m * gy, dsy, gs));
            }
        }
        if (act && sub == 0) {
            if (!MS && g.softmax) {
                // logit gradient w_k (d/dw_k - sum_j w_j d/dw_j); d/dw_k was
                // staged in grec (rounded to T)
                for (int k = 0; k < g.K; ++k)
                    grec[3 * k + 2] = Elem<T>::from_f(sn.weight(Elem<T>::to_f(rec[3 * k + 2])) *
                                                      (Elem<T>::to_f(grec[3 * k + 2]) - dotw));
            }
            if (MS) {
                const float raw = Elem<T>::to_f(static_cast<const T *>(ms.raw)[pr]);
                graw[pr] = Elem<T>::from_f(gs == 0.0f ? 0.0f : gs * msdcn_scale_grad(raw, ms.s0[grp], ms.smax));
            }
        }
    }
}

}  // namespace dcn4
