// dcn4_fwd.cuh -- forward kernels of DCNv4 and its groupwise multi-scale
// variant (MSDCN).
//
// Operation (DCNv4 paper digest "(论文速读）DCNv4：高效可变形卷积算子", sections
// "移除Softmax归一化" and "方法1. 消除冗余工作负载"; FlowDCN article "2.2 DCN结构简介"
// and "3.1 组间多尺度可变形卷积"): out[p0, g*D + d] = sum_k m_k * bilinear(in, p0 +
// p_k + dp_k)[g*D + d], with the D channels of a group sharing the offsets and
// weights, and for MSDCN dp_k = s_g(p0) * dir_k.
//
// Two kernels here (the vectorised global-memory one is in dcn4_bwd_vec.cuh):
//  * fwd_generic_kernel: one thread per (pixel, group, run of <= 8 channels),
//    scalar loads straight from global memory. Any shape, any alignment.
//  * fwd_halo_kernel: one thread per (pixel, group) covering all D channels.
//    A CTA owns an output tile x a slice of Gc groups. One TMA tile load
//    brings the input window the tile can reach (tile +- R pixels, zeros
//    outside the image by the TMA out-of-bounds fill) into shared memory, and
//    a second TMA tile copy (or, when the pixel stride rules that out,
//    per-pixel bulk copies) brings the tile's offset/weight records. Every corner gather
//    is then a 16-byte shared-memory load; samples that leave the window use
//    16-byte global loads instead. Lanes rotate the order of their 16-byte
//    chunks so that the 8 lanes of each shared-memory phase hit 8 different
//    bank quads whatever pixel they sample (the pixel stride is a multiple of
//    128 bytes), which keeps random gathers free of bank conflicts.
#pragma once

#include "dcn4_common.cuh"

namespace dcn4 {

// The device error word (defined once, in dcn4_kernels.cu, before this file).


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
        if (!DCN4_GMEM_OK(rec, g.K * 3 * sizeof(T), ow, ow_bytes_of(g, sizeof(T)))) continue;
        float s = 1.0f;
        if (MS) {
            const T *rp = static_cast<const T *>(ms.raw) + pix * g.G + grp;
            const float raw = DCN4_GMEM_OK(rp, sizeof(T), ms.raw, raw_bytes(g, sizeof(T)))
                                  ? Elem<T>::to_f(*rp) : 0.0f;
            s = msdcn_scale(raw, ms.s0[grp], ms.smax);
        }
        SoftmaxNorm sn{0.0f, 1.0f};
        if (!MS && g.softmax) {
            float mx = -INFINITY, sum = 0.0f;
            for (int k = 0; k < g.K; ++k) mx = fmaxf(mx, Elem<T>::to_f(rec[3 * k + 2]));
            for (int k = 0; k < g.K; ++k) sum += expf(Elem<T>::to_f(rec[3 * k + 2]) - mx);
            sn = SoftmaxNorm{mx, 1.0f / sum};
        }
        float acc[CH];
#pragma unroll
        for (int d = 0; d < CH; ++d) acc[d] = 0.0f;
        const T *src = in + (size_t)n * img + (size_t)grp * g.D + d0;
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
#pragma unroll
                for (int a = 0; a < 2; ++a) {
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int yy = y0 + a, xx = x0 + b;
                        if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) continue;
                        const float w = (a ? ly : 1.0f - ly) * (b ? lx : 1.0f - lx) * m;
                        const T *p = src + ((size_t)yy * g.W + xx) * g.C;
                        if (!DCN4_GMEM_OK(p, cnt * sizeof(T), in, input_bytes(g, sizeof(T))))
                            continue;
#pragma unroll
                        for (int d = 0; d < CH; ++d)
                            if (d < cnt) acc[d] = fmaf(w, Elem<T>::to_f(p[d]), acc[d]);
                    }
                }
            }
        }
        T *dst = out + (size_t)pix * g.C + (size_t)grp * g.D + d0;
        if (!DCN4_GMEM_OK(dst, cnt * sizeof(T), out, output_bytes(g, sizeof(T)))) continue;
#pragma unroll
        for (int d = 0; d < CH; ++d)
            if (d < cnt) dst[d] = Elem<T>::from_f(acc[d]);
    }
}

// ------------------------------------------------------------------------
// Shared-memory halo kernel (3x3 taps, D*sizeof(T) = 16*U bytes)
// ------------------------------------------------------------------------

// Shared-memory byte layout of one halo CTA: STAGES x (window, record
// slots), each stage a multiple of 128 bytes, then the mbarriers.
struct HaloSmem {
    static __host__ __device__ __forceinline__ int stage_bytes(const HaloPlan &p) {
        return (p.halo_bytes + p.TH * p.TW * p.slot_bytes + 127) / 128 * 128;
    }
    // + the win and empty barriers of every stage and one record barrier per
    // warp (up to 16) and stage
    static __host__ __device__ __forceinline__ int total_bytes(const HaloPlan &p, int stages) {
        return stages * stage_bytes(p) + 8 * stages * (2 + 16);
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

// One output tile of the halo kernel: image n, groups [g0, g0+Gc), output
// rows [ho0, ho0+th_eff) and columns [wo0, wo0+tw_eff); the staged window
// starts at image row hy0, column hx0.
struct TileCoord {
    int n, g0, ho0, wo0, hy0, hx0, th_eff, tw_eff;
    unsigned long long gp0;  // flat output pixel index of (n, ho0, wo0)
};

__device__ __forceinline__ TileCoord tile_coord(int t, const Geometry &g, const HaloPlan &pl) {
    TileCoord c;
    const int tw = t % pl.tiles_w;
    t /= pl.tiles_w;
    const int th = t % pl.tiles_h;
    t /= pl.tiles_h;
    const int sl = t % pl.slices;
    c.n = t / pl.slices;
    c.ho0 = th * pl.TH;
    c.wo0 = tw * pl.TW;
    c.g0 = sl * pl.Gc;
    c.hy0 = pl.full_h ? -1 : c.ho0 * g.sh - g.ph - pl.R;
    c.hx0 = pl.full_w ? -1 : c.wo0 * g.sw - g.pw - pl.R;
    c.th_eff = min(pl.TH, g.Ho - c.ho0);
    c.tw_eff = min(pl.TW, g.Wo - c.wo0);
    c.gp0 = ((unsigned long long)c.n * g.Ho + c.ho0) * g.Wo + c.wo0;
    return c;
}

// Bulk-copies into their slots the records of the tile pixels whose pairs
// this warp computes: with NT threads and LPP lanes per pair, thread t
// handles pairs t/LPP, (t + NT)/LPP, ..., so warp w owns pixel blocks
// [(32w + k*NT)/(LPP*Gc), +32/(LPP*Gc)) for k = 0, 1, ...
// Completes on `bar` (arrival count 1); all 32 lanes call it, lane l copies
// pixel l of each block it has, lane 0 arrives with the warp's byte count.
template <typename T, int LPP = 1>
__device__ __forceinline__ void stage_records(const TileCoord &tc, const Geometry &g,
                                              const HaloPlan &pl, const T *__restrict__ ow,
                                              unsigned long long ow_bytes, unsigned char *slots,
                                              int nt, uint32_t bar, const unsigned char *sbase) {
    (void)sbase;
    constexpr int EB = Elem<T>::kBytes;
    constexpr unsigned long long REC = 27ull * EB;
    const int lane = threadIdx.x & 31;
    const int npix = pl.TH * pl.TW;
    const bool mine = lane < ((32 / LPP) >> pl.lgGc);
    auto span = [&](int p, unsigned long long &a, unsigned long long &e,
                    unsigned long long &end) -> bool {
        const int ty = p >> pl.lgTW, tx_ = p & (pl.TW - 1);
        if (p >= npix || ty >= tc.th_eff || tx_ >= tc.tw_eff) return false;
        const unsigned long long gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx_;
        const unsigned long long start = (gp * g.G + tc.g0) * REC;
        end = start + (unsigned long long)pl.Gc * REC;
        a = start & ~15ull;
        e = min((end + 15ull) & ~15ull, ow_bytes & ~15ull);
        return true;
    };
    uint32_t tx = 0;
    for (int base = ((threadIdx.x & ~31) / LPP) >> pl.lgGc; base < npix;
         base += (nt / LPP) >> pl.lgGc) {
        const int p = base + lane;
        unsigned long long a, e, end;
        if (!mine || !span(p, a, e, end)) continue;
        if (e > a) tx += (uint32_t)(e - a);
        // the tensor's last bytes when its size is not a multiple of 16
        unsigned char *slot = slots + (size_t)p * pl.slot_bytes;
        for (unsigned long long q = e; q < end; q += EB) {
            const unsigned char *sp = reinterpret_cast<const unsigned char *>(ow) + q;
            if (!DCN4_GMEM_OK(sp, EB, ow, ow_bytes) || !DCN4_SMEM_OK(slot + (q - a), EB, sbase))
                continue;
            if (EB == 4)
                *reinterpret_cast<unsigned *>(slot + (q - a)) = *reinterpret_cast<const unsigned *>(sp);
            else
                *reinterpret_cast<unsigned short *>(slot + (q - a)) =
                    *reinterpret_cast<const unsigned short *>(sp);
        }
    }
    uint32_t total = tx;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    // order the warp's earlier generic reads of these slots (and the tail
    // stores above) before the async-proxy writes and the arrive
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive_expect_tx(bar, total);
    __syncwarp();
    for (int base = ((threadIdx.x & ~31) / LPP) >> pl.lgGc; base < npix;
         base += (nt / LPP) >> pl.lgGc) {
        const int p = base + lane;
        unsigned long long a, e, end;
        if (!mine || !span(p, a, e, end) || e <= a) continue;
        if (!DCN4_SMEM_OK(slots + (size_t)p * pl.slot_bytes, (unsigned)(e - a), sbase) ||
            !DCN4_GMEM_OK(reinterpret_cast<const unsigned char *>(ow) + a, (unsigned)(e - a), ow,
                          ow_bytes))
            continue;
        bulk_load(smem_u32(slots + (size_t)p * pl.slot_bytes),
                  reinterpret_cast<const unsigned char *>(ow) + a, (uint32_t)(e - a), bar);
    }
}

// TMA load of a tile's input window into `halo`, completing on `bar`
// (arrival count 1); called by one thread.
__device__ __forceinline__ void stage_window(const TileCoord &tc, const CUtensorMap *tmap,
                                             const Geometry &g, const HaloPlan &pl, int eb,
                                             unsigned char *halo, uint32_t bar,
                                             const unsigned char *sbase) {
    (void)sbase;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint32_t wbytes = (uint32_t)pl.HR * pl.HC * pl.Gc * g.D * eb;
    mbar_arrive_expect_tx(bar, wbytes);
    if (DCN4_SMEM_OK(halo, wbytes, sbase))
        tma_load_4d(smem_u32(halo), tmap, tc.g0 * g.D, tc.hx0, tc.hy0, tc.n, bar);
}

// With pl.rec_tma: the tile's input window and its records ([TH][TW]
// x rec_box elements from the 16-byte boundary at or below the slice's first
// value; zero fill past the image) on one barrier; called by one thread.
__device__ __forceinline__ void stage_window_records(const TileCoord &tc, const CUtensorMap *tmap,
                                                     const CUtensorMap *tmap_ow, const Geometry &g,
                                                     const HaloPlan &pl, int eb,
                                                     unsigned char *halo, unsigned char *slots,
                                                     uint32_t bar, const unsigned char *sbase) {
    (void)sbase;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint32_t wbytes = (uint32_t)pl.HR * pl.HC * pl.Gc * g.D * eb;
    const uint32_t rbytes = (uint32_t)pl.TH * pl.TW * pl.rec_box * eb;
    mbar_arrive_expect_tx(bar, wbytes + rbytes);
    if (DCN4_SMEM_OK(halo, wbytes, sbase))
        tma_load_4d(smem_u32(halo), tmap, tc.g0 * g.D, tc.hx0, tc.hy0, tc.n, bar);
    const int x0 = (tc.g0 * 27) & ~(16 / eb - 1);
    if (DCN4_SMEM_OK(slots, rbytes, sbase))
        tma_load_4d(smem_u32(slots), tmap_ow, x0, tc.wo0, tc.ho0, tc.n, bar);
}

// The gathers of one staged tile: LPP lanes per (pixel, group), each with
// U/LPP of its 16-byte chunks (one lane with all of them when LPP = 1). With
// DEF (LPP = 1) and el.entries set, a pair with escaped taps appends an
// EscList entry (slot from the CTA's counter *esc_n) instead of loading them.
template <typename T, int U, bool MS, int MV, int LPP, bool DEF = false>
__device__ __forceinline__ void compute_tile(const TileCoord &tc, const Geometry &g,
                                             const HaloPlan &pl, const T *__restrict__ in,
                                             T *__restrict__ out, const MsdcnParams &ms,
                                             const unsigned char *halo,
                                             const unsigned char *slots, int ct, int nct,
                                             const unsigned char *sbase,
                                             const EscList &el = EscList{},
                                             int *esc_n = nullptr) {
    static_assert(!DEF || LPP == 1, "deferred escapes take one lane per pair");
    (void)sbase;
    constexpr int EB = Elem<T>::kBytes;
    constexpr int VE = Elem<T>::kPerVec;  // elements per 16-byte chunk
    constexpr int REC = 27 * EB;          // bytes of one (pixel, group) record
    constexpr int PS = 128;               // bytes per staged pixel (Gc*D*EB, host-checked)
    const int D = g.D;
    const int RS = pl.HC * PS;            // bytes per staged row
    const int lane = threadIdx.x & 31;
    const int npairs = pl.TH * pl.TW * pl.Gc;
    const size_t img = (size_t)g.H * g.W * g.C;
    // the staged window in image coordinates: corners x0, x0+1 are inside iff
    // hx_lo <= x < hx_hi (NaN fails the test and goes to the escape path)
    const float hx_lo = (float)tc.hx0, hx_hi = (float)(tc.hx0 + pl.HC - 1);
    const float hy_lo = (float)tc.hy0, hy_hi = (float)(tc.hy0 + pl.HR - 1);
    const float PSf = (float)PS, RSf = (float)RS;
    const float dwf = (float)g.dw, dhf = (float)g.dh;
    constexpr int UL = U / LPP;  // chunks of this lane
    // nct is a multiple of LPP, so a thread keeps its lane-in-pair `sub`
    for (int t = ct; t < npairs * LPP; t += nct) {
        const int f = t / LPP, sub = t & (LPP - 1);
        const int pix = f >> pl.lgGc;
        const int gl = f & (pl.Gc - 1);
        const int ty = pix >> pl.lgTW, tx = pix & (pl.TW - 1);
        if (ty >= tc.th_eff || tx >= tc.tw_eff) continue;
        const int ho = tc.ho0 + ty, wo = tc.wo0 + tx;
        const unsigned long long gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx;
        // the record's offset within its 16-byte-aligned copy (arithmetic mod
        // 2^32); records written in place (rec_tma == 2) start their slot
        const unsigned mis =
            pl.rec_tma == 2 ? 0u
            : pl.rec_tma    ? ((unsigned)(tc.g0 * 27) & (unsigned)(16 / EB - 1)) * (unsigned)EB
                            : ((unsigned)gp * (unsigned)g.G + (unsigned)tc.g0) * (unsigned)REC & 15u;
        const unsigned char *rec = slots + (size_t)pix * pl.slot_bytes + mis + gl * REC;
        // the reader takes whole words from the record's 4-byte boundary
        if (!DCN4_SMEM_OK(reinterpret_cast<const unsigned char *>(
                              reinterpret_cast<uintptr_t>(rec) & ~uintptr_t(3)),
                          EB == 4 ? 108u : 60u, sbase))
            continue;
        float v[27];
        RecordReader<T>::read(rec, v);
        float s = 1.0f;
        const bool dil = MS && g.msd_dil;
        if (MS) {
            const T *rp = static_cast<const T *>(ms.raw) + gp * g.G + tc.g0 + gl;
            const float raw = DCN4_GMEM_OK(rp, EB, ms.raw, raw_bytes(g, EB)) ? Elem<T>::to_f(*rp)
                                                                              : 0.0f;
            s = msdcn_scale(raw, ms.s0[tc.g0 + gl], ms.smax);
            if (!dil) {
#pragma unroll
                for (int k = 0; k < 9; ++k) {
                    v[3 * k] = __fmul_rn(s, v[3 * k]);
                    v[3 * k + 1] = __fmul_rn(s, v[3 * k + 1]);
                }
            }
        }
        SoftmaxNorm sn{0.0f, 1.0f};
        if (!MS && g.softmax) {
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
        // chunk rotation: the 8 lanes of a shared-memory phase start at
        // different 16-byte chunks, so their loads hit 8 different bank quads
        const int r = (LPP == 1) ? ((U <= 8) ? (((lane & 7) * U) >> 3) : (f & (U - 1)))
                                 : ((lane / LPP) & (UL - 1));
        // this lane's c-th chunk
        auto chunk = [&](int c) -> int { return sub * UL + ((c + r) & (UL - 1)); };
        const unsigned char *row0[UL], *row1[UL];
#pragma unroll
        for (int c = 0; c < UL; ++c) {
            row0[c] = halo + (size_t)gl * D * EB + chunk(c) * 16;
            row1[c] = row0[c] + RS;
        }
        float acc[UL][VE];
#pragma unroll
        for (int c = 0; c < UL; ++c)
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[c][e] = 0.0f;

        const float fbx = (float)(wo * g.sw - g.pw), fby = (float)(ho * g.sh - g.ph);
        const float bxs[3] = {fbx, fbx + dwf, fbx + 2.0f * dwf};
        const float bys[3] = {fby, fby + dhf, fby + 2.0f * dhf};
        unsigned esc = 0;
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            float x, y;
            if (dil) {  // centre + s * (grid offset + dir * os)
                x = __fadd_rn(bxs[1], __fmul_rn(s, __fadd_rn((float)(k % 3 - 1) * dwf,
                                                              __fmul_rn(v[3 * k], g.os))));
                y = __fadd_rn(bys[1], __fmul_rn(s, __fadd_rn((float)(k / 3 - 1) * dhf,
                                                              __fmul_rn(v[3 * k + 1], g.os))));
            } else {
                x = __fadd_rn(bxs[k % 3], __fmul_rn(v[3 * k], g.os));
                y = __fadd_rn(bys[k / 3], __fmul_rn(v[3 * k + 1], g.os));
            }
            const float m = v[3 * k + 2];
            if (x >= hx_lo && x < hx_hi && y >= hy_lo && y < hy_hi) {
                const float x0f = floorf(x), y0f = floorf(y);
                const float lx = x - x0f, ly = y - y0f;
                const float mly = m * ly, mhy = m - mly;
                const float w01 = mhy * lx, w00 = mhy - w01;
                const float w11 = mly * lx, w10 = mly - w11;
                // integer-valued floats below 2^24: the byte offset is exact
                const int off = __float2int_rz(fmaf(y0f - hy_lo, RSf, (x0f - hx_lo) * PSf));
#pragma unroll
                for (int c = 0; c < UL; ++c) {
                    const unsigned char *a0 = row0[c] + off;
                    const unsigned char *a1 = row1[c] + off;
                    const uint4 q00 = DCN4_LDS16(a0, sbase);
                    const uint4 q01 = DCN4_LDS16(a0 + PS, sbase);
                    const uint4 q10 = DCN4_LDS16(a1, sbase);
                    const uint4 q11 = DCN4_LDS16(a1 + PS, sbase);
                    if (MV == 2) {
                        VecMathPacked<T>::blend4(acc[c], q00, q01, q10, q11, w00, w01, w10, w11);
                    } else if (MV == 1) {
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
        if (DEF && esc != 0u && el.entries != nullptr) {
            const int slot = atomicAdd(esc_n, 1);
            if (slot < el.cap) {
                unsigned char *e =
                    el.entries + ((size_t)blockIdx.x * el.cap + slot) * (size_t)el.entry_bytes;
                const unsigned long long P = gp * g.G + tc.g0 + gl;
                if (DCN4_GMEM_OK(e, (unsigned)el.entry_bytes, el.entries, el.bytes)) {
                    *reinterpret_cast<uint4 *>(e) =
                        make_uint4((unsigned)P, (unsigned)(P >> 32), esc, 0u);
                    float4 *pf = reinterpret_cast<float4 *>(e + 16);
#pragma unroll
                    for (int c = 0; c < UL; ++c)
#pragma unroll
                        for (int q = 0; q < VE; q += 4)
                            pf[(chunk(c) * VE + q) >> 2] =
                                make_float4(acc[c][q], acc[c][q + 1], acc[c][q + 2], acc[c][q + 3]);
                }
                continue;
            }
        }
        // samples outside the staged window (rare): 16-byte loads from global
        // memory, each corner tested against the image
        const T *gbase = in + (size_t)tc.n * img + (size_t)(tc.g0 + gl) * D;
        while (esc) {
            const int k = __ffs(esc) - 1;
            esc &= esc - 1;
            float dx, dy, m;
            record_tap<T>(rec, k, dx, dy, m);  // inside the record checked above
            if (!MS && g.softmax) m = sn.weight(m);
            const int i = k / 3, j = k - 3 * (k / 3);
            float x, y, dsx, dsy;
            if (MS) {
                x = msdcn_coord(dil, wo * g.sw - g.pw, j, 3, g.dw, s, dx, g.os, &dsx);
                y = msdcn_coord(dil, ho * g.sh - g.ph, i, 3, g.dh, s, dy, g.os, &dsy);
            } else {
                x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
                y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
            }
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
                for (int c = 0; c < UL; ++c)
                    VecMath<T>::fma(acc[c], DCN4_LDG16(p + chunk(c), in, input_bytes(g, EB)), wc[q]);
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + gp * g.C + (size_t)(tc.g0 + gl) * D);
#pragma unroll
        for (int c = 0; c < UL; ++c)
            if (DCN4_GMEM_OK(dst + chunk(c), 16, out, output_bytes(g, EB)))
                dst[chunk(c)] = VecMath<T>::pack(acc[c]);
    }
}

// One deferred escape (an EscList entry of the staged forward): starts from
// the entry's partial sums and adds the escaped taps in ascending order with
// the staged kernel's own arithmetic (the pair's record read again from
// global memory; position, softmax weight or MSDCN scale, corner weights,
// fp32 multiply-adds of 16-byte global loads, out-of-image corners skipped),
// then writes the pair's output: the in-place result, bit for bit.
template <typename T, int U, bool MS>
__device__ __forceinline__ void finish_escape(const unsigned char *e, const Geometry &g,
                                              const T *__restrict__ in,
                                              const T *__restrict__ ow, T *__restrict__ out,
                                              const MsdcnParams &ms) {
    constexpr int EB = Elem<T>::kBytes;
    constexpr int VE = Elem<T>::kPerVec;
    const size_t img = (size_t)g.H * g.W * g.C;
    const unsigned long long npairs = (unsigned long long)g.N * g.Ho * g.Wo * g.G;
    const unsigned long long in_b = input_bytes(g, EB), out_b = output_bytes(g, EB);
    const unsigned long long ow_b = npairs * 27 * EB;
    (void)in_b, (void)out_b, (void)ow_b, (void)npairs;
    const uint4 meta = *reinterpret_cast<const uint4 *>(e);
    const unsigned long long P = meta.x | ((unsigned long long)meta.y << 32);
    const unsigned esc = meta.z;
    if (!DCN4_CHECK(P < npairs)) return;
    const T *rec = ow + P * 27;
    if (!DCN4_GMEM_OK(rec, 27 * EB, ow, ow_b)) return;
    float acc[U][VE];
    const float4 *pf = reinterpret_cast<const float4 *>(e + 16);
#pragma unroll
    for (int c = 0; c < U; ++c)
#pragma unroll
        for (int q = 0; q < VE / 4; ++q) {
            const float4 f = pf[c * (VE / 4) + q];
            acc[c][4 * q] = f.x, acc[c][4 * q + 1] = f.y;
            acc[c][4 * q + 2] = f.z, acc[c][4 * q + 3] = f.w;
        }
    const int gg = (int)(P % (unsigned)g.G);
    const unsigned long long gp = P / (unsigned)g.G;
    const int wo = (int)(gp % (unsigned)g.Wo);
    const unsigned long long rr = gp / (unsigned)g.Wo;
    const int ho = (int)(rr % (unsigned)g.Ho), n = (int)(rr / (unsigned)g.Ho);
    float s = 1.0f;
    const bool dil = MS && g.msd_dil;
    if (MS) {
        const T *rp = static_cast<const T *>(ms.raw) + P;
        const float raw = DCN4_GMEM_OK(rp, EB, ms.raw, raw_bytes(g, EB))
                              ? Elem<T>::to_f(*rp) : 0.0f;
        s = msdcn_scale(raw, ms.s0[gg], ms.smax);
    }
    SoftmaxNorm sn{0.0f, 1.0f};
    if (!MS && g.softmax) {
        float mx = Elem<T>::to_f(rec[2]);
#pragma unroll
        for (int k = 1; k < 9; ++k) mx = fmaxf(mx, Elem<T>::to_f(rec[3 * k + 2]));
        float sum = 0.0f;
#pragma unroll
        for (int k = 0; k < 9; ++k) sum += expf(Elem<T>::to_f(rec[3 * k + 2]) - mx);
        sn = SoftmaxNorm{mx, 1.0f / sum};
    }
    const T *gbase = in + (size_t)n * img + (size_t)gg * g.D;
    // tap k: its corner weights and which corners lie in the image (none
    // when the sample is outside), loads into qv
    auto tap = [&](int k, float *wc, bool *ok, uint4 (*qv)[U]) {
        const float dx = Elem<T>::to_f(rec[3 * k]), dy = Elem<T>::to_f(rec[3 * k + 1]);
        float m = Elem<T>::to_f(rec[3 * k + 2]);
        if (!MS && g.softmax) m = sn.weight(m);
        const int i = k / 3, j = k - 3 * i;
        float x, y, dsx, dsy;
        if (MS) {
            x = msdcn_coord(dil, wo * g.sw - g.pw, j, 3, g.dw, s, dx, g.os, &dsx);
            y = msdcn_coord(dil, ho * g.sh - g.ph, i, 3, g.dh, s, dy, g.os, &dsy);
        } else {
            x = sample_coord(wo * g.sw - g.pw + j * g.dw, dx, g.os);
            y = sample_coord(ho * g.sh - g.ph + i * g.dh, dy, g.os);
        }
        const bool inside = x > -1.0f && x < (float)g.W && y > -1.0f && y < (float)g.H;
        const float x0f = floorf(x), y0f = floorf(y);
        const float lx = x - x0f, ly = y - y0f;
        const float mly = m * ly, mhy = m - mly;
        const float w01 = mhy * lx, w11 = mly * lx;
        wc[0] = mhy - w01, wc[1] = w01, wc[2] = mly - w11, wc[3] = w11;
        const int x0 = inside ? (int)x0f : 0, y0 = inside ? (int)y0f : 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int yy = y0 + (q >> 1), xx = x0 + (q & 1);
            ok[q] = inside && yy >= 0 && yy < g.H && xx >= 0 && xx < g.W;
            const uint4 *p =
                reinterpret_cast<const uint4 *>(gbase + ((size_t)yy * g.W + xx) * g.C);
#pragma unroll
            for (int c = 0; c < U; ++c)
                qv[q][c] = ok[q] ? DCN4_LDG16(p + c, in, in_b) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    unsigned em = esc & 0x1ffu;
    while (em) {
        const int k = __ffs(em) - 1;
        em &= em - 1;
        float wc[4];
        bool ok[4];
        uint4 qv[4][U];
        tap(k, wc, ok, qv);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (ok[q])
#pragma unroll
                for (int c = 0; c < U; ++c) VecMath<T>::fma(acc[c], qv[q][c], wc[q]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + gp * g.C + (size_t)gg * g.D);
#pragma unroll
    for (int c = 0; c < U; ++c)
        if (DCN4_GMEM_OK(dst + c, 16, out, out_b)) dst[c] = VecMath<T>::pack(acc[c]);
}

// Persistent halo kernel. CTA b handles tiles b, b + gridDim.x, ...; thread
// t of the NW warps owns (pixel, group) pairs t, t + 32NW, ... of every tile.
// The input window (and, with pl.rec_tma, the tile's records) is shared:
// warp 0 loads it (win[s]) once every warp has released the buffer
// (empty[s], NW arrivals). Without pl.rec_tma each warp consumes the records
// of its own tile pixels: it bulk-copies those itself and waits on its own
// barrier (rec[w][s]). With STAGES == 2 the copies of
// the next tile are in flight while the current one is computed. Every wait
// is bounded; on expiry the warp sets the error word, lets its own copies in
// flight land and returns.
template <typename T, int U, bool MS, int MV, int STAGES, int NW, int LPP>
__global__ void __launch_bounds__(NW * 32, 1)
fwd_halo_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap_ow,
                Geometry g, HaloPlan pl, const T *__restrict__ in, const T *__restrict__ ow,
                T *__restrict__ out, unsigned long long ow_bytes,
                const __grid_constant__ MsdcnParams ms, const __grid_constant__ EscList el) {
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ int esc_n;  // deferred escapes: entries taken
    const int stage_bytes = HaloSmem::stage_bytes(pl);
    const uint32_t win0 = smem_u32(smem + STAGES * stage_bytes);  // win[s]   at +8s
    const uint32_t empty0 = win0 + 8 * STAGES;                     // empty[s] at +8s
    const uint32_t rec0 = empty0 + 8 * STAGES;                     // rec[w][s] at +8(w*STAGES+s)
    const int ntiles = g.N * pl.slices * pl.tiles_h * pl.tiles_w;
    const int warp = threadIdx.x >> 5;
    const bool leader = (threadIdx.x & 31) == 0;
    const uint32_t myrec = rec0 + 8 * (warp * STAGES);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(win0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, NW);
        }
        for (int b = 0; b < NW * STAGES; ++b) mbar_init(rec0 + 8 * b, 1);
        fence_barrier_init();
        esc_n = 0;
    }
    __syncthreads();

    // window of the CTA's k-th tile (coordinates tc), once every warp has
    // released its stage
    auto window = [&](const TileCoord &tc, int k) -> bool {
        const int s = k % STAGES, use = k / STAGES;
        if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1, kWaitLimitNs)) return false;
        if (leader) {
            unsigned char *buf = smem + s * stage_bytes;
            if (pl.rec_tma)
                stage_window_records(tc, &tmap, &tmap_ow, g, pl, Elem<T>::kBytes, buf,
                                     buf + pl.halo_bytes, win0 + 8 * s, smem);
            else
                stage_window(tc, &tmap, g, pl, Elem<T>::kBytes, buf, win0 + 8 * s, smem);
        }
        return true;
    };
    // per-warp record copies (the records of the warp's own pairs), unless
    // they come with the window
    auto records = [&](const TileCoord &tc, int k) {
        if (pl.rec_tma) return;
        const int s = k % STAGES;
        stage_records<T, LPP>(tc, g, pl, ow, ow_bytes, smem + s * stage_bytes + pl.halo_bytes, NW * 32,
                         myrec + 8 * s, smem);
    };
    auto records_ready = [&](int k) -> bool {
        return pl.rec_tma ||
               mbar_wait_bounded(myrec + 8 * (k % STAGES), (k / STAGES) & 1, kWaitLimitNs);
    };
    // on an expired wait: let this warp's copies of tiles k0..k1 land
    auto drain = [&](int k0, int k1, bool with_window) {
        for (int k = k0 < 0 ? 0 : k0; k <= k1; ++k) {
            records_ready(k);
            if (with_window)
                mbar_wait_bounded(win0 + 8 * (k % STAGES), (k / STAGES) & 1, kWaitLimitNs);
        }
    };

    TileCoord cur;
    if ((int)blockIdx.x < ntiles) {
        cur = tile_coord(blockIdx.x, g, pl);
        records(cur, 0);
        if (warp == 0) window(cur, 0);
    }
    int i = 0;
    bool bail = false;  // this warp stopped on an expired wait
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
        const int s = i % STAGES;
        const int tn = t + gridDim.x;
        TileCoord nxt;
        if (tn < ntiles) nxt = tile_coord(tn, g, pl);
        int issued = i;
        if (STAGES == 2 && tn < ntiles) {
            records(nxt, i + 1);
            if (warp == 0 && !window(nxt, i + 1)) {
                if (leader) atomicOr(&g_error_word, kErrTimeout);
                drain(i, i + 1, false);
                drain(i, i, true);
                bail = true;
                break;
            }
            issued = i + 1;
        }
        const bool ok = mbar_wait_bounded(win0 + 8 * s, (i / STAGES) & 1, kWaitLimitNs) &&
                        records_ready(i);
        if (!ok) {
            if (leader) atomicOr(&g_error_word, kErrTimeout);
            drain(i, issued, warp == 0);
            bail = true;
            break;
        }
        const unsigned char *buf = smem + s * stage_bytes;
        compute_tile<T, U, MS, MV, LPP, LPP == 1>(cur, g, pl, in, out, ms, buf,
                                                 buf + pl.halo_bytes, threadIdx.x, NW * 32, smem,
                                                 el, &esc_n);
        __syncwarp();
        if (leader) mbar_arrive(empty0 + 8 * s);
        if (STAGES == 1 && tn < ntiles) {
            records(nxt, i + 1);
            if (warp == 0 && !window(nxt, i + 1)) {
                if (leader) atomicOr(&g_error_word, kErrTimeout);
                drain(i + 1, i + 1, false);
                bail = true;
                break;
            }
        }
        cur = nxt;
    }
    // the CTA's deferred escapes, once every warp is done with its tiles
    // (every warp gets here: each wait is bounded); none after an expired wait
    if (LPP == 1 && el.entries != nullptr) {
        if (__syncthreads_or(bail)) return;
        const int ne = min(esc_n, el.cap);
        for (int ei = threadIdx.x; ei < ne; ei += NW * 32) {
            const unsigned char *e =
                el.entries + ((size_t)blockIdx.x * el.cap + ei) * (size_t)el.entry_bytes;
            if (DCN4_GMEM_OK(e, (unsigned)el.entry_bytes, el.entries, el.bytes))
                finish_escape<T, U, MS>(e, g, in, ow, out, ms);
        }
    }
}

}  // namespace dcn4
