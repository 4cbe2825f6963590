// dcn4_bwd_halo.cuh -- shared-memory backward kernel of DCNv4 (3x3 taps,
// 128-byte staged pixels). Included after dcn4_fwd.cuh (shares its tile
// geometry, record reader and staging conventions).
//
// The forward is out[p0, g*D+d] = sum_k m_k sum_c w_c in[corner_c, g*D+d]
// (DCNv4 digest "方法1. 消除冗余工作负载"; FlowDCN "2.2"). Its gradients:
//   d/dm_k  = sum_c w_c <go, V_c>,       d/ddx_k = os m_k sum_c (dw_c/dlx) <go, V_c>,
//   d/ddy_k = os m_k sum_c (dw_c/dly) <go, V_c>,   grad_in[corner_c] += m_k w_c go.
// The first three are gathers (like the forward). The last is a scatter;
// scattering with per-element shared-memory atomics would cost 16 atomic
// lane-operations per corner, so the kernel transposes instead: it sorts the
// CTA's samples by destination cell (one integer atomic per sample), and each
// (staged pixel, group) then gathers the contributions of the four cells it
// is a corner of, accumulating in registers, and adds the sum to grad_input
// with 16-byte vector reductions (neighbouring tiles' windows overlap): packed
// 16-bit reductions into the 16-bit grad_input itself (DIRECT), else fp32
// reductions into the workspace.
//
// One CTA per (image, output tile, group slice); NW warps; phases:
//   stage  TMA: input window + grad_out tile (+ records when the pixel stride
//          allows a TMA tile copy); else bulk copies of the records
//   A      per (pixel, group): corner gathers, the three gradients per tap,
//          count each staged sample into its cell (rank = atomic result)
//   B      exclusive scan of the cell counts
//   C      per (pixel, group): write each staged sample's record at
//          offset[cell] + rank, over the window buffer (no longer needed)
//   E      copy the staged grad_offset_weight out with coalesced stores
//   D      per (staged pixel, group): gather from its four cells, flush
// Samples outside the staged window take a global path with atomics.
#pragma once

#include "dcn4_fwd.cuh"

namespace dcn4 {

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// Adds 8 packed 16-bit values (one 16-byte vector of T) to global memory.
template <typename T> struct Red16;
template <> struct Red16<__nv_bfloat16> {
    static __device__ __forceinline__ void add(void *p, const uint4 &v) {
        asm volatile("red.global.add.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x),
                     "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    }
};
template <> struct Red16<__half> {
    static __device__ __forceinline__ void add(void *p, const uint4 &v) {
        asm volatile("red.global.add.noftz.v4.f16x2 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x),
                     "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    }
};
template <> struct Red16<float> {
    static __device__ __forceinline__ void add(void *, const uint4 &) {}
};

// Unpacks a 16-byte chunk of T into fp32.
template <typename T> struct ChunkUnpack;
template <> struct ChunkUnpack<float> {
    static __device__ __forceinline__ void get(const uint4 &v, float *o) {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    }
};
template <> struct ChunkUnpack<__nv_bfloat16> {
    static __device__ __forceinline__ void get(const uint4 &v, float *o) {
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o[2 * e] = __uint_as_float(w[e] << 16);
            o[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
};
template <> struct ChunkUnpack<__half> {
    static __device__ __forceinline__ void get(const uint4 &v, float *o) {
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[e]));
            o[2 * e] = f.x;
            o[2 * e + 1] = f.y;
        }
    }
};

// <a, b> where a is one 16-byte chunk of T and b the same channels already
// unpacked to fp32 (grad_out, unpacked once per pair). For 16-bit T every
// product of two stored values is exact in fp32 (8- or 11-bit significands);
// the sums are fp32, even channels in .x, odd ones in .y.
template <typename T> struct DotF;
template <> struct DotF<float> {
    static __device__ __forceinline__ float dot(const uint4 &a, const float *b) {
        float s0 = __uint_as_float(a.x) * b[0];
        float s1 = __uint_as_float(a.y) * b[1];
        s0 = fmaf(__uint_as_float(a.z), b[2], s0);
        s1 = fmaf(__uint_as_float(a.w), b[3], s1);
        return s0 + s1;
    }
};
template <> struct DotF<__nv_bfloat16> {
    static __device__ __forceinline__ float dot(const uint4 &a, const float *b) {
        const unsigned w[4] = {a.x, a.y, a.z, a.w};
        float2 s = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            s = __ffma2_rn(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u)),
                           make_float2(b[2 * e], b[2 * e + 1]), s);
        return s.x + s.y;
    }
};
template <> struct DotF<__half> {
    static __device__ __forceinline__ float dot(const uint4 &a, const float *b) {
        const unsigned w[4] = {a.x, a.y, a.z, a.w};
        float2 s = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            s = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2 *>(&w[e])),
                           make_float2(b[2 * e], b[2 * e + 1]), s);
        return s.x + s.y;
    }
};

// <a, b> with both chunks packed 16-bit: the sm_100 mixed-precision fma
// (exact 16x16-bit products, fp32 sums); fp32 falls back to DotF.
template <typename T> struct PackedDotM {
    static __device__ __forceinline__ float dot(const uint4 &a, const uint4 &b) {
        float bf[4] = {__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z),
                       __uint_as_float(b.w)};
        return DotF<float>::dot(a, bf);
    }
};
#define DCN4_PDOT(TY)                                                                          \
    static __device__ __forceinline__ float dot(const uint4 &a, const uint4 &b) {              \
        const unsigned wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};             \
        float s0 = 0.f, s1 = 0.f;                                                              \
        _Pragma("unroll") for (int e = 0; e < 4; ++e) {                                        \
            asm("{ .reg .b16 al, ah, bl, bh; mov.b32 {al, ah}, %2; mov.b32 {bl, bh}, %3;"      \
                " fma.rn.f32." TY " %0, al, bl, %0; fma.rn.f32." TY " %1, ah, bh, %1; }"       \
                : "+f"(s0), "+f"(s1) : "r"(wa[e]), "r"(wb[e]));                              \
        }                                                                                      \
        return s0 + s1;                                                                        \
    }
template <> struct PackedDotM<__nv_bfloat16> { DCN4_PDOT("bf16") };
template <> struct PackedDotM<__half> { DCN4_PDOT("f16") };
#undef DCN4_PDOT

// Block-wide exclusive scan of counts[0..n) in place; counts[n] = total.
template <int NW>
__device__ __forceinline__ void block_exclusive_scan(int *counts, int n, int *warp_sums) {
    const int NT = NW * 32;
    const int per = (n + NT - 1) / NT;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += counts[i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < NW) warp_sums[lane] = wi - w;  // exclusive warp prefix
        if (lane == NW - 1) warp_sums[NW] = wi;   // total
    }
    __syncthreads();
    int run = warp_sums[warp] + incl - local;
    for (int i = lo; i < hi; ++i) {
        const int c = counts[i];
        counts[i] = run;
        run += c;
    }
    if (threadIdx.x == 0) counts[n] = warp_sums[NW];
    __syncthreads();
}

// DIRECT: grad_input (16-bit T) accumulates in place: each CTA's fp32 sums
// are rounded once to T and added with packed 16-bit reductions (no fp32
// workspace). Otherwise sums go to the fp32 workspace `gacc`.
// MS: the FlowDCN multi-scale variant ("3.1"): ow holds (dir_x, dir_y, m),
// the offset is s * dir with s from scale_raw (ms.raw); grad_offset_weight
// receives d/d dir and graw the gradient of scale_raw, as in
// bwd_generic_kernel.
template <typename T, int U, int NW, bool MIXED, bool DIRECT, bool MS>
__global__ void __launch_bounds__(NW * 32, 512 / (NW * 32))
bwd_halo_kernel(const __grid_constant__ CUtensorMap tmap_in,
                const __grid_constant__ CUtensorMap tmap_go,
                const __grid_constant__ CUtensorMap tmap_ow, Geometry g, HaloPlan pl,
                BwdLayout L, const T *__restrict__ in, const T *__restrict__ ow,
                T *__restrict__ gow, float *__restrict__ gacc, T *__restrict__ gin,
                unsigned long long ow_bytes, const __grid_constant__ MsdcnParams ms,
                T *__restrict__ graw) {
    constexpr int EB = Elem<T>::kBytes;
    constexpr int VE = Elem<T>::kPerVec;
    constexpr int REC = 27 * EB;
    constexpr int PS = 128;
    constexpr int NT = NW * 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ int warp_sums[NW + 1];
    unsigned char *halo = smem;
    unsigned char *gotile = smem + L.go_off;
    unsigned char *slots = smem + L.slots_off;
    T *gows = reinterpret_cast<T *>(smem + L.gows_off);
    int *counts = reinterpret_cast<int *>(smem + L.counts_off);
    const uint32_t bar = smem_u32(smem + L.bar_off);
    // sorted sample records (lx, ly, m, byte offset of the source grad_out
    // vector), written over the window and record slots after phase A
    float4 *srec = reinterpret_cast<float4 *>(smem);
    // DIRECT (16-bit weights, 16-bit grad_input): 8-byte records instead,
    // {bf16 (1-ly)*m | bf16 ly*m, fp16 lx | grad_out offset / 16}: the owner
    // gather reads them at random addresses, where bytes are the cost
    constexpr bool CR = DIRECT && sizeof(T) == 2;
    uint2 *srec8 = reinterpret_cast<uint2 *>(smem);

    const TileCoord tc = tile_coord(blockIdx.x, g, pl);
    const int D = g.D;
    const int RS = pl.HC * PS;
    const int lane = threadIdx.x & 31;
    const size_t img = (size_t)g.H * g.W * g.C;

    // ---------------- stage ----------------
    if (threadIdx.x == 0) {
        mbar_init(bar, NT);
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= L.ncells; i += NT) counts[i] = 0;
    __syncthreads();
    {
        uint32_t tx = 0;
        if (threadIdx.x == 0)
            tx = (uint32_t)pl.HR * pl.HC * PS + (uint32_t)pl.TH * pl.TW * PS +
                 (pl.rec_tma ? (uint32_t)pl.TH * pl.TW * pl.rec_box * EB : 0u);
        const int npix = pl.rec_tma ? 0 : pl.TH * pl.TW;  // per-pixel copies
        for (int p = threadIdx.x; p < npix; p += NT) {
            const int ty = p >> pl.lgTW, tx_ = p & (pl.TW - 1);
            if (ty >= tc.th_eff || tx_ >= tc.tw_eff) continue;
            const unsigned long long gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx_;
            const unsigned long long start = (gp * g.G + tc.g0) * (unsigned long long)REC;
            const unsigned long long end = start + (unsigned long long)pl.Gc * REC;
            const unsigned long long a = start & ~15ull;
            const unsigned long long e = min((end + 15ull) & ~15ull, ow_bytes & ~15ull);
            if (e > a) tx += (uint32_t)(e - a);
            unsigned char *slot = slots + (size_t)p * pl.slot_bytes;
            for (unsigned long long q = e; q < end; q += EB) {
                const unsigned char *sp = reinterpret_cast<const unsigned char *>(ow) + q;
                if (EB == 4)
                    *reinterpret_cast<unsigned *>(slot + (q - a)) = *reinterpret_cast<const unsigned *>(sp);
                else
                    *reinterpret_cast<unsigned short *>(slot + (q - a)) =
                        *reinterpret_cast<const unsigned short *>(sp);
            }
        }
        mbar_arrive_expect_tx(bar, tx);
        if (threadIdx.x == 0) {
            tma_load_4d(smem_u32(halo), &tmap_in, tc.g0 * D, tc.hx0, tc.hy0, tc.n, bar);
            tma_load_4d(smem_u32(gotile), &tmap_go, tc.g0 * D, tc.wo0, tc.ho0, tc.n, bar);
            if (pl.rec_tma)
                tma_load_4d(smem_u32(slots), &tmap_ow, (tc.g0 * 27) & ~(16 / EB - 1), tc.wo0, tc.ho0,
                            tc.n, bar);
        }
        for (int p = threadIdx.x; p < npix; p += NT) {
            const int ty = p >> pl.lgTW, tx_ = p & (pl.TW - 1);
            if (ty >= tc.th_eff || tx_ >= tc.tw_eff) continue;
            const unsigned long long gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx_;
            const unsigned long long start = (gp * g.G + tc.g0) * (unsigned long long)REC;
            const unsigned long long end = start + (unsigned long long)pl.Gc * REC;
            const unsigned long long a = start & ~15ull;
            const unsigned long long e = min((end + 15ull) & ~15ull, ow_bytes & ~15ull);
            if (e > a)
                bulk_load(smem_u32(slots + (size_t)p * pl.slot_bytes),
                          reinterpret_cast<const unsigned char *>(ow) + a, (uint32_t)(e - a), bar);
        }
    }
    const bool ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
        if (threadIdx.x == 0) atomicOr(&g_error_word, kErrTimeout);
        mbar_wait_bounded(bar, 0, kWaitLimitNs);
        return;
    }

    // ---------------- A: gradients of offsets and weights; cell counts ----------------
    const float hx_lo = (float)tc.hx0, hx_hi = (float)(tc.hx0 + pl.HC - 1);
    const float hy_lo = (float)tc.hy0, hy_hi = (float)(tc.hy0 + pl.HR - 1);
    const float PSf = (float)PS, RSf = (float)RS;
    const float dwf = (float)g.dw, dhf = (float)g.dh;
    const int npairs = pl.TH * pl.TW * pl.Gc;
    const int cells_w = pl.HC - 1;
    const int ncpg = (pl.HR - 1) * cells_w;  // cells per group; cell = gl * ncpg + y * cells_w + x
    unsigned kr[9];          // (cell << 16) | rank of each staged tap; 0xffffffff otherwise
    float v[27];
    int f = threadIdx.x;
    const bool has_pair = f < npairs;
    int pix = 0, gl = 0, ho = 0, wo = 0;
    bool valid = false;
    unsigned long long gp = 0;
    unsigned start = 0;  // the record's offset within its 16-byte-aligned copy
    if (has_pair) {
        pix = f >> pl.lgGc;
        gl = f & (pl.Gc - 1);
        const int ty = pix >> pl.lgTW, tx = pix & (pl.TW - 1);
        valid = ty < tc.th_eff && tx < tc.tw_eff;
        ho = tc.ho0 + ty;
        wo = tc.wo0 + tx;
        gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx;
        start = pl.rec_tma ? ((unsigned)(tc.g0 * 27) & (unsigned)(16 / EB - 1)) * (unsigned)EB
                           : ((unsigned)gp * (unsigned)g.G + (unsigned)tc.g0) * (unsigned)REC & 15u;
    }
#pragma unroll
    for (int k = 0; k < 9; ++k) kr[k] = 0xffffffffu;
    const int r = (U <= 8) ? (((lane & 7) * U) >> 3) : (f & (U - 1));
    float s = 1.0f, gs = 0.0f;  // MSDCN scale of this (pixel, group), d/ds
    if (valid) {
        const unsigned char *rec = slots + (size_t)pix * pl.slot_bytes + start + gl * REC;
        RecordReader<T>::read(rec, v);
        if (MS)
            s = msdcn_scale(Elem<T>::to_f(static_cast<const T *>(ms.raw)[gp * g.G + tc.g0 + gl]),
                            ms.s0[tc.g0 + gl], ms.smax);
        // DCNv3 weights: softmax of the logits over the taps; the logit
        // gradient w_k (gw_k - sum_j w_j gw_j) is formed after the taps from
        // the staged gw_k
        SoftmaxNorm sn{0.0f, 1.0f};
        if (g.softmax) {
            float mx = v[2];
#pragma unroll
            for (int k = 1; k < 9; ++k) mx = fmaxf(mx, v[3 * k + 2]);
            float sum = 0.0f;
#pragma unroll
            for (int k = 0; k < 9; ++k) {
                v[3 * k + 2] = expf(v[3 * k + 2] - mx);
                sum += v[3 * k + 2];
            }
            const float inv = 1.0f / sum;
#pragma unroll
            for (int k = 0; k < 9; ++k) v[3 * k + 2] *= inv;
            sn = SoftmaxNorm{mx, inv};
        }
        float dotw = 0.0f;
        const unsigned char *row0[U], *row1[U];
        // gof[c]: this pair's grad_out chunk (c + r) mod U, unpacked to fp32;
        // gop[c] the same chunk packed
        float gof[U][VE];
        uint4 gop[U];
#pragma unroll
        for (int c = 0; c < U; ++c) {
            const int cc = (c + r) & (U - 1);
            row0[c] = halo + (size_t)gl * D * EB + cc * 16;
            row1[c] = row0[c] + RS;
            gop[c] = *reinterpret_cast<const uint4 *>(gotile + (size_t)pix * PS + gl * D * EB + cc * 16);
            ChunkUnpack<T>::get(gop[c], gof[c]);
        }
        const float fbx = (float)(wo * g.sw - g.pw), fby = (float)(ho * g.sh - g.ph);
        const float bxs[3] = {fbx, fbx + dwf, fbx + 2.0f * dwf};
        const float bys[3] = {fby, fby + dhf, fby + 2.0f * dhf};
        T *gout_rec = gows + ((size_t)pix * pl.Gc + gl) * 27;
        unsigned esc = 0;
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            float x, y, dsx = 0.f, dsy = 0.f;  // ds*: d position / d s (MSDCN)
            if (MS) {
                x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, k % 3, 3, g.dw, s, v[3 * k], g.os, &dsx);
                y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, k / 3, 3, g.dh, s, v[3 * k + 1], g.os,
                                &dsy);
            } else {
                x = __fadd_rn(bxs[k % 3], __fmul_rn(v[3 * k], g.os));
                y = __fadd_rn(bys[k / 3], __fmul_rn(v[3 * k + 1], g.os));
            }
            const float m = v[3 * k + 2];
            float gx = 0.f, gy = 0.f, gm = 0.f;
            // a sample outside (-1, W) x (-1, H) has no gradient and no
            // contribution (checked explicitly: at x == -1 exactly the window
            // would otherwise give a one-sided d/dx from the corner x0 + 1)
            const bool inside = x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H;
            if (!inside) {
                // nothing to do
            } else if (x >= hx_lo && x < hx_hi && y >= hy_lo && y < hy_hi) {
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const float hx = 1.0f - lx, hy = 1.0f - ly;
                const int off = __float2int_rz(fmaf(y0f - hy_lo, RSf, (x0f - hx_lo) * PSf));
                float d00 = 0.f, d01 = 0.f, d10 = 0.f, d11 = 0.f;
#pragma unroll
                for (int c = 0; c < U; ++c) {
                    const unsigned char *a0 = row0[c] + off;
                    const unsigned char *a1 = row1[c] + off;
                    d00 += PackedDotM<T>::dot(*reinterpret_cast<const uint4 *>(a0), gop[c]);
                    d01 += PackedDotM<T>::dot(*reinterpret_cast<const uint4 *>(a0 + PS), gop[c]);
                    d10 += PackedDotM<T>::dot(*reinterpret_cast<const uint4 *>(a1), gop[c]);
                    d11 += PackedDotM<T>::dot(*reinterpret_cast<const uint4 *>(a1 + PS), gop[c]);
                }
                gm = hy * (hx * d00 + lx * d01) + ly * (hx * d10 + lx * d11);
                const float px = hy * (d01 - d00) + ly * (d11 - d10);  // d/d position
                const float py = hx * (d10 - d00) + lx * (d11 - d01);
                gx = g.os * m * px;
                gy = g.os * m * py;
                if (MS) gs = fmaf(m * px, dsx, fmaf(m * py, dsy, gs));
                const int cell = gl * ncpg + ((int)(y0f - hy_lo)) * cells_w + (int)(x0f - hx_lo);
                const int rank = atomicAdd(&counts[cell], 1);
                kr[k] = ((unsigned)cell << 16) | (unsigned)rank;
            } else {
                esc |= 1u << k;
            }
            gout_rec[3 * k] = Elem<T>::from_f(MS && gx != 0.f ? s * gx : gx);
            gout_rec[3 * k + 1] = Elem<T>::from_f(MS && gy != 0.f ? s * gy : gy);
            gout_rec[3 * k + 2] = Elem<T>::from_f(gm);
            dotw = fmaf(m, gm, dotw);
        }
        // samples outside the staged window: global gathers, fp32 atomics
        const T *gsrc = in + (size_t)tc.n * img + (size_t)(tc.g0 + gl) * D;
        float *gdst = gacc + (size_t)tc.n * img + (size_t)(tc.g0 + gl) * D;
        while (esc) {
            const int k = __ffs(esc) - 1;
            esc &= esc - 1;
            const int i = k / 3, j = k - 3 * (k / 3);
            float dx, dy, m;
            record_tap<T>(rec, k, dx, dy, m);
            if (g.softmax) m = sn.weight(m);
            float x, y, dsx = 0.f, dsy = 0.f;
            if (MS) {
                x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, j, 3, g.dw, s, dx, g.os, &dsx);
                y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, i, 3, g.dh, s, dy, g.os, &dsy);
            } else {
                x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
            }
            float gx = 0.f, gy = 0.f, gm = 0.f;
            if (x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H) {
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const int x0 = (int)x0f, y0 = (int)y0f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int a = q >> 1, b = q & 1;
                    const int yy = y0 + a, xx = x0 + b;
                    if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                    const float wy = a ? ly : 1.0f - ly, wx = b ? lx : 1.0f - lx;
                    const size_t at = ((size_t)yy * g.W + xx) * g.C;
                    const uint4 *p = reinterpret_cast<const uint4 *>(gsrc + at);
                    float dot = 0.f;
#pragma unroll
                    for (int c = 0; c < U; ++c) dot += DotF<T>::dot(__ldg(p + ((c + r) & (U - 1))), gof[c]);
                    gm = fmaf(wy * wx, dot, gm);
                    gx = fmaf(b ? wy : -wy, dot, gx);
                    gy = fmaf(a ? wx : -wx, dot, gy);
                    const float cw = m * wy * wx;
#pragma unroll
                    for (int c = 0; c < U; ++c) {
                        const int cc = (c + r) & (U - 1);
                        float go[VE];
#pragma unroll
                        for (int d = 0; d < VE; ++d) go[d] = cw * gof[c][d];
                        if (DIRECT) {
                            Red16<T>::add(gin + (size_t)tc.n * img + (size_t)(tc.g0 + gl) * D + at +
                                              cc * VE,
                                          VecMath<T>::pack(go));
                        } else {
#pragma unroll
                            for (int d = 0; d < VE; ++d) atomicAdd(gdst + at + cc * VE + d, go[d]);
                        }
                    }
                }
                if (MS) gs = fmaf(m * gx, dsx, fmaf(m * gy, dsy, gs));
                gx *= g.os * m;
                gy *= g.os * m;
            }
            gout_rec[3 * k] = Elem<T>::from_f(MS && gx != 0.f ? s * gx : gx);
            gout_rec[3 * k + 1] = Elem<T>::from_f(MS && gy != 0.f ? s * gy : gy);
            gout_rec[3 * k + 2] = Elem<T>::from_f(gm);
            dotw = fmaf(m, gm, dotw);
        }
        if (MS) {
            const float raw = Elem<T>::to_f(static_cast<const T *>(ms.raw)[gp * g.G + tc.g0 + gl]);
            graw[gp * g.G + tc.g0 + gl] = Elem<T>::from_f(
                gs == 0.0f ? 0.0f : gs * msdcn_scale_grad(raw, ms.s0[tc.g0 + gl], ms.smax));
        }
        if (g.softmax) {
#pragma unroll
            for (int k = 0; k < 9; ++k)
                gout_rec[3 * k + 2] =
                    Elem<T>::from_f(v[3 * k + 2] * (Elem<T>::to_f(gout_rec[3 * k + 2]) - dotw));
        }
    }
    __syncthreads();  // window reads, counts and gows staging complete

    // ---------------- B: cell offsets ----------------
    block_exclusive_scan<NW>(counts, L.ncells, warp_sums);

    // ---------------- C: sorted sample records (over the window) ----------------
    if (valid) {
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            if (kr[k] == 0xffffffffu) continue;
            const int cell = (int)(kr[k] >> 16), rank = (int)(kr[k] & 0xffffu);
            const int i = k / 3, j = k - 3 * (k / 3);
            float x, y;
            if (MS) {
                float dsx, dsy;
                x = msdcn_coord(g.msd_dil, wo * g.sw - g.pw, j, 3, g.dw, s, v[3 * k], g.os, &dsx);
                y = msdcn_coord(g.msd_dil, ho * g.sh - g.ph, i, 3, g.dh, s, v[3 * k + 1], g.os, &dsy);
            } else {
                x = sample_coord(wo * g.sw - g.pw + j * g.dw, v[3 * k], g.os);
                y = sample_coord(ho * g.sh - g.ph + i * g.dh, v[3 * k + 1], g.os);
            }
            const int pos = counts[cell] + rank;
            const float lx = x - floorf(x), ly = y - floorf(y), m = v[3 * k + 2];
            const unsigned goff = (unsigned)(pix * PS + gl * D * EB);
            if (CR) {
                const __nv_bfloat162 wy2 = __floats2bfloat162_rn(m - ly * m, ly * m);
                srec8[pos] = make_uint2(*reinterpret_cast<const unsigned *>(&wy2),
                                        (unsigned)__half_as_ushort(__float2half_rn(lx)) |
                                            ((goff >> 4) << 16));
            } else {
                srec[pos] = make_float4(lx, ly, m, __uint_as_float(goff));
            }
        }
    }
    __syncthreads();

    // ---------------- E: grad_offset_weight out (one warp per pixel) ----------------
    {
        const int npix = pl.TH * pl.TW;
        const int span = pl.Gc * 27 * EB;  // bytes per pixel, contiguous in gow
        for (int p = threadIdx.x >> 5; p < npix; p += NW) {
            const int ty = p >> pl.lgTW, tx = p & (pl.TW - 1);
            if (ty >= tc.th_eff || tx >= tc.tw_eff) continue;
            const unsigned long long q = tc.gp0 + (unsigned long long)ty * g.Wo + tx;
            unsigned char *dst = reinterpret_cast<unsigned char *>(gow + (q * g.G + tc.g0) * 27);
            const unsigned char *src = reinterpret_cast<const unsigned char *>(gows) + (size_t)p * span;
            // widest word that divides both addresses and the span
            const unsigned al = (unsigned)(reinterpret_cast<uintptr_t>(dst) |
                                           reinterpret_cast<uintptr_t>(src) | (uintptr_t)span);
            if ((al & 7) == 0) {
                for (int e = lane * 8; e < span; e += 256)
                    *reinterpret_cast<uint2 *>(dst + e) = *reinterpret_cast<const uint2 *>(src + e);
            } else if ((al & 3) == 0) {
                for (int e = lane * 4; e < span; e += 128)
                    *reinterpret_cast<unsigned *>(dst + e) = *reinterpret_cast<const unsigned *>(src + e);
            } else {
                for (int e = lane * EB; e < span; e += 32 * EB)
                    *reinterpret_cast<T *>(dst + e) = *reinterpret_cast<const T *>(src + e);
            }
        }
    }

    // ---------------- D: gather per (staged pixel, group) and flush ----------------
    const int nown = pl.HR * pl.HC * pl.Gc;
    for (int o = threadIdx.x; o < nown; o += NT) {
        const int ogl = o & (pl.Gc - 1);
        const int q = o >> pl.lgGc;
        const int qy = (int)__umulhi((unsigned)q, L.hc_magic), qx = q - qy * pl.HC;
        const int iy = tc.hy0 + qy, ix = tc.hx0 + qx;
        if (iy < 0 || iy >= g.H || ix < 0 || ix >= g.W) continue;
        const int rr = (U <= 8) ? (((lane & 7) * U) >> 3) : (o & (U - 1));
        float acc[U][VE];
#pragma unroll
        for (int c = 0; c < U; ++c)
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[c][e] = 0.0f;
        // cells are numbered group-major, so for each corner row a the two
        // cells (cy, qx - 1) (corner b = 1) and (cy, qx) (b = 0) are adjacent
        // and their entries form one contiguous range split at es
        bool any = false;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const int cy = qy - a;
            if (cy < 0 || cy >= pl.HR - 1) continue;
            const int row = ogl * ncpg + cy * cells_w;
            const int e0 = counts[row + max(qx - 1, 0)];
            const int es = counts[row + min(qx, cells_w)];
            const int e1 = counts[row + min(qx, cells_w - 1) + 1];
            any |= e1 > e0;
            for (int e = e0; e < e1; ++e) {
                float w;
                const unsigned char *gsrc;
                if (CR) {
                    const uint2 r = srec8[e];
                    const float wy = __uint_as_float(a ? (r.x & 0xffff0000u) : (r.x << 16));
                    const float lx = __half2float(__ushort_as_half((unsigned short)(r.y & 0xffffu)));
                    w = wy * (e < es ? lx : 1.0f - lx);
                    gsrc = gotile + ((r.y >> 16) << 4);
                } else {
                    const float4 rec4 = srec[e];
                    const float wy = a ? rec4.y : 1.0f - rec4.y;
                    const float wx = e < es ? rec4.x : 1.0f - rec4.x;
                    w = wy * wx * rec4.z;
                    gsrc = gotile + __float_as_uint(rec4.w);
                }
#pragma unroll
                for (int c = 0; c < U; ++c) {
                    const int cc = (c + rr) & (U - 1);
                    const uint4 q = *reinterpret_cast<const uint4 *>(gsrc + cc * 16);
                    if (MIXED)
                        VecMathMixed<T>::fma(acc[c], q, w);
                    else
                        VecMath<T>::fma(acc[c], q, w);
                }
            }
        }
        if (any) {
            const size_t at = (size_t)tc.n * img + ((size_t)iy * g.W + ix) * g.C +
                              (size_t)(tc.g0 + ogl) * D;
#pragma unroll
            for (int c = 0; c < U; ++c) {
                const int cc = (c + rr) & (U - 1);
                if (DIRECT) {
                    Red16<T>::add(gin + at + cc * VE, VecMath<T>::pack(acc[c]));
                } else {
#pragma unroll
                    for (int e = 0; e < VE; e += 4)
                        red_add_v4(gacc + at + cc * VE + e, acc[c][e], acc[c][e + 1],
                                   acc[c][e + 2], acc[c][e + 3]);
                }
            }
        }
    }
}

}  // namespace dcn4
