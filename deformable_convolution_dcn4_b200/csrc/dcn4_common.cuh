// dcn4_common.cuh -- shared device helpers and launch parameter blocks for the
// DCNv4 / MSDCN kernels (sm_100a). Host and device code both include it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcn4 {

// Bits of the device error word (read back by dcn4_last_device_error).
constexpr unsigned kErrTimeout = 1u;   // a bounded mbarrier wait expired
constexpr unsigned kErrInternal = 2u;  // a consistency check failed
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per wait

constexpr int kMaxGroups = 1024;
constexpr int kMaxTaps = 64;  // kh * kw

// Problem geometry, copied into every launch.
struct Geometry {
    int N, H, W, C, G, D;
    int kh, kw, K;
    int sh, sw, ph, pw, dh, dw;
    int Ho, Wo;
    float os;     // offset_scale
    int softmax;  // DCNv3 weights: softmax of m over the K taps
    int msd_dil;  // MSDCN scale-as-dilation reading
};

// Tile of the generic producer kernel: pixels x outputs per CTA, channels
// per shared-memory chunk.
constexpr int kProducerPixels = 128;
constexpr int kProducerOuts = 128;
constexpr int kProducerK = 16;

// Shape of one producer launch.
struct ProducerGeo {
    int N, H, W, C;
    int J;   // outputs per pixel, G * kh * kw * 3
    int NP;  // J rounded up to a multiple of 16 (tensor-core N)
    long long npix;
    int ntiles;  // 128-pixel tiles (tensor-core kernel)
};

// Shared-memory carve-up of the tensor-core producer kernel (byte offsets).
struct ProducerTcLayout {
    int b_off, a_off, x_off, x_bytes, x_nbuf, dwf_off, dwt_off, linb_off, row_off, bar_off,
        bytes, tmem_cols;

    // x_nbuf staged pixel ranges: 2 (the next tile's copy overlaps this
    // tile's work) or 1 (it overlaps only the MMA and the epilogue)
    static ProducerTcLayout make(int C, int J, int NP, int W, int x_nbuf) {
        (void)J;
        ProducerTcLayout L;
        L.b_off = 0;                     // lin_w, NP rows x C (core matrices)
        L.a_off = L.b_off + NP * C * 2;  // h, 128 rows x C (core matrices)
        L.x_off = L.a_off + 128 * C * 2;  // staged pixel ranges
        L.x_bytes = ((128 + 2 * W + 2) * C * 2 + 127) / 128 * 128;
        L.x_nbuf = x_nbuf;
        L.dwf_off = L.x_off + x_nbuf * L.x_bytes;  // fp32 dw_w [9][C], dw_b [C]
        L.dwt_off = L.dwf_off + 10 * C * 4;   // dw_w [9][C] in the data type
        L.linb_off = L.dwt_off + (9 * C * 2 + 15) / 16 * 16;  // fp32 lin_b [NP]
        L.row_off = (L.linb_off + NP * 4 + 15) / 16 * 16;  // int2 (y, x) per tile row
        L.bar_off = L.row_off + 128 * 8;                     // 3 mbarriers, tmem address
        L.bytes = L.bar_off + 32;
        int cols = 32;
        while (cols < NP) cols <<= 1;
        L.tmem_cols = cols;
        return L;
    }
};

// MSDCN extras: per-group scale priors travel inside the launch parameters.
// s = min(s0 * softplus(raw), smax), softplus(r) = max(r, 0) + log1p(exp(-|r|)).
__device__ __forceinline__ float msdcn_scale(float raw, float s0, float smax) {
    float sp = __fadd_rn(fmaxf(raw, 0.0f), log1pf(expf(-fabsf(raw))));
    float s = __fmul_rn(s0, sp);
    return (s > smax) ? smax : s;
}

// d s / d raw for the scale above: s0 * sigmoid(raw) (sigmoid is the
// derivative of softplus) while s0 * softplus(raw) <= smax, the branch
// msdcn_scale keeps; 0 once the clamp is active or raw is NaN.
__device__ __forceinline__ float msdcn_scale_grad(float raw, float s0, float smax) {
    const float sp = __fadd_rn(fmaxf(raw, 0.0f), log1pf(expf(-fabsf(raw))));
    const float u = __fmul_rn(s0, sp);
    if (!(u <= smax)) return 0.0f;
    return s0 / (1.0f + expf(-raw));
}

struct MsdcnParams {
    const void *raw;  // [N][Ho][Wo][G] in the element type
    float smax;
    float s0[kMaxGroups];
};

// Shared-memory layout of the backward halo kernel (chosen on the host);
// all offsets in bytes from the start of dynamic shared memory.
struct BwdLayout {
    int go_off;       // grad_out tile, TH*TW pixels x 128 bytes
    int slots_off;    // offset/weight records, TH*TW slots
    int gows_off;     // grad_offset_weight staging, TH*TW*Gc*27 elements
    int counts_off;   // ncells + 1 ints: per-cell sample counts, then offsets
    int bar_off;      // one mbarrier
    int ncells;       // (HR-1)*(HC-1)*Gc destination cells
    int max_samples;  // TH*TW*Gc*9; sorted sample records reuse the window
    int olist_off;    // owner list (u16 per owner, sorted by sample count), a u16 rank and
                      // a u8 count per owner, after the sorted samples
    unsigned hc_magic;  // ceil(2^32 / HC): q / HC == __umulhi(q, hc_magic) for q < 2^16
    int smem_bytes;
    int threads;      // 256 (two CTAs per SM) or 512
    int lpp;          // lanes per (pixel, group): 1, or 4 for 8 chunks (128-byte groups)
};

// Tiling of the shared-memory halo kernels (chosen on the host).
struct HaloPlan {
    int TH, TW;          // output tile (TW a power of two)
    int Gc;              // groups per CTA (a power of two dividing G)
    int lgTW, lgGc;      // log2(TW), log2(Gc)
    int R;               // offset reach covered by the halo, in pixels
    int HR, HC;          // halo rows / columns held in shared memory
    int full_h, full_w;  // 1: the halo is the whole image plus a 1-pixel zero border
    int tiles_h, tiles_w, slices;
    int slot_bytes;      // bytes per output pixel of staged offset/weight triples
    int halo_bytes;      // HR*HC*Gc*D*elem, rounded up to 128
    int stages;          // 2: double-buffered pipeline, 1: single buffer
    int smem_bytes;      // dynamic shared memory of one CTA
    int rec_tma;         // 1: records arrive by one TMA tile copy per tile (forward);
                         // 2: the fused kernel writes them, slot-aligned, in place
    int rec_box;         // elements per pixel of that copy (Gc*27 plus alignment slack)
};

// Deferred escapes of the staged forward (chosen on the host). A (pixel,
// group) pair with taps outside the staged window does not wait for their
// global loads: it leaves an entry here, and the CTA adds those taps and
// writes the pair's output after its last tile, with all its warps busy on
// such entries. Entry layout, entry_bytes = 16 + 4*D:
//   bytes 0-7    pair index P = ((n*Ho + ho)*Wo + wo)*G + g   (u64)
//   bytes 8-11   mask of the escaped taps (bit k: tap k)
//   bytes 16-    the in-window partial sums, D fp32 values in channel order
// CTA b of the staged kernel appends to entries [b*cap, (b+1)*cap) while
// it works through its tiles, and finishes them itself once all its warps
// are done; once its region is full it handles further escapes in place.
struct EscList {
    unsigned char *entries;    // nullptr: every escape handled in place
    int cap;                   // entries per CTA
    int entry_bytes;
    unsigned long long bytes;  // of the entries area (bounds of the checked build)
};

// Tiling and shared-memory carve-up of the 2-D tiled tensor-core producer
// (byte offsets from the start of dynamic shared memory; chosen on the host).
struct ProducerTc2dLayout {
    int TH, TW, lgTW;      // pixel tile (TW a power of two, TH * TW <= 128)
    int tiles_h, tiles_w;  // tiles per image
    int x_off, x_bytes;    // x neighbourhood of a tile, (TH+2) x (TW+2) pixels x C
    int a_off;             // depthwise outputs: 128 rows x C, tcgen05 core matrices
    int b_off;             // lin_w: NP rows x C, core matrices (rows >= J zero)
    int o_off;             // the tile's outputs, TH*TW rows of J values (TMA store source)
    int dwt_off;           // dw_weight [9][C] in the data type
    int dwb_off;           // dw_bias [C] in fp32
    int linb_off;          // lin_bias [NP] in fp32 (zero past J)
    int bar_off;           // two mbarriers and the tensor-memory address
    int bytes;             // dynamic shared memory of one CTA
    int tmem_cols;         // a power of two >= NP, >= 32
};

// Shared-memory carve-up of the fused producer + forward kernel (byte offsets
// from the start of dynamic shared memory; chosen on the host).
struct FusedLayout {
    int win_off;    // input window of the tile's group slice (HaloPlan::halo_bytes)
    int slots_off;  // the tile's records, TH*TW slots of HaloPlan::slot_bytes
    int x_off;      // x neighbourhood of the tile, (TH+2) x (TW+2) pixels x C
    int x_bytes;    // bytes of that copy
    int a_off;      // depthwise outputs: 128 rows x C, tcgen05 K-major core matrices
    int b_off;      // the slice's rows of lin_weight: NP rows x C, core matrices
    int dwt_off;    // dw_weight [9][C] in the data type
    int dwb_off;    // dw_bias [C] in fp32
    int linb_off;   // the slice's lin_bias [NP] in fp32 (zero past JS)
    int bar_off;    // three mbarriers and the tensor-memory address
    int bytes;      // dynamic shared memory of one CTA
    int JS;         // outputs of one slice, Gc * 27
    int NP;         // JS rounded up to 16 (the MMA's N)
    int tmem_cols;  // tensor-memory columns allocated: a power of two >= NP, >= 32
};

// Byte sizes of the tensors of one call (bounds of the checked build).
__host__ __device__ __forceinline__ unsigned long long input_bytes(const Geometry &g, int eb) {
    return (unsigned long long)g.N * g.H * g.W * g.C * eb;
}
__host__ __device__ __forceinline__ unsigned long long output_bytes(const Geometry &g, int eb) {
    return (unsigned long long)g.N * g.Ho * g.Wo * g.C * eb;
}
__host__ __device__ __forceinline__ unsigned long long ow_bytes_of(const Geometry &g, int eb) {
    return (unsigned long long)g.N * g.Ho * g.Wo * g.G * g.K * 3 * eb;
}
__host__ __device__ __forceinline__ unsigned long long raw_bytes(const Geometry &g, int eb) {
    return (unsigned long long)g.N * g.Ho * g.Wo * g.G * eb;
}

// ---- element types -------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    static constexpr int kPerVec = 4;  // elements per 16-byte vector
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr int kPerVec = 8;
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Elem<__half> {
    static constexpr int kBytes = 2;
    static constexpr int kPerVec = 8;
    static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
    static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};

// ---- sample position: fp32, product and sum rounded separately -------------
__device__ __forceinline__ float sample_coord(int base, float delta, float os) {
    return __fadd_rn((float)base, __fmul_rn(delta, os));
}

// MSDCN sample coordinate along one axis for tap index t (j along W, i along
// H) of a window of `kt` taps with dilation `dil`, output base
// `base` = o*stride - pad, scale s and direction d:
//   scale-as-offset  base + t*dil + (s*d)*os
//   scale-as-dilation  c + s*(p_t + d*os), c = base + (kt-1)/2 * dil the
//                      window centre, p_t = (t - (kt-1)/2) * dil
// (each product and sum rounded to fp32). *ds receives d coord / d s.
__device__ __forceinline__ float msdcn_coord(bool dilation, int base, int t, int kt, int dil,
                                             float s, float d, float os, float *ds) {
    if (!dilation) {
        *ds = __fmul_rn(d, os);
        return sample_coord(base + t * dil, __fmul_rn(s, d), os);
    }
    const float c = (float)base + 0.5f * (float)((kt - 1) * dil);
    const float p = ((float)t - 0.5f * (float)(kt - 1)) * (float)dil;
    const float u = __fadd_rn(p, __fmul_rn(d, os));
    *ds = u;
    return __fadd_rn(c, __fmul_rn(s, u));
}

// DCNv3 weights: softmax over the K logits m of one (pixel, group); the
// weight of logit m is expf(m - mx) * inv.
struct SoftmaxNorm {
    float mx, inv;
    __device__ __forceinline__ float weight(float m) const { return expf(m - mx) * inv; }
};

// ---- fp32 accumulation of 16-byte vectors -------------------------------
// acc[0..kPerVec) += w * (16-byte vector v of T), fp32 arithmetic, using the
// sm_100 packed fp32 pair fma (__ffma2_rn) on channel pairs.
__device__ __forceinline__ void ffma2(float &a0, float &a1, float x0, float x1, float w) {
    const float2 r = __ffma2_rn(make_float2(x0, x1), make_float2(w, w), make_float2(a0, a1));
    a0 = r.x;
    a1 = r.y;
}

template <typename T> struct VecMath;
template <> struct VecMath<float> {
    static __device__ __forceinline__ void fma(float *acc, const uint4 &v, float w) {
        ffma2(acc[0], acc[1], __uint_as_float(v.x), __uint_as_float(v.y), w);
        ffma2(acc[2], acc[3], __uint_as_float(v.z), __uint_as_float(v.w), w);
    }
    static __device__ __forceinline__ uint4 pack(const float *a) {
        return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]),
                          __float_as_uint(a[2]), __float_as_uint(a[3]));
    }
};
template <> struct VecMath<__nv_bfloat16> {
    static __device__ __forceinline__ void fma2w(float *acc, unsigned w2, float w) {
        ffma2(acc[0], acc[1], __uint_as_float(w2 << 16), __uint_as_float(w2 & 0xffff0000u), w);
    }
    static __device__ __forceinline__ void fma(float *acc, const uint4 &v, float w) {
        fma2w(acc + 0, v.x, w);
        fma2w(acc + 2, v.y, w);
        fma2w(acc + 4, v.z, w);
        fma2w(acc + 6, v.w, w);
    }
    static __device__ __forceinline__ unsigned pk(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<unsigned *>(&h);
    }
    static __device__ __forceinline__ uint4 pack(const float *a) {
        return make_uint4(pk(a[0], a[1]), pk(a[2], a[3]), pk(a[4], a[5]), pk(a[6], a[7]));
    }
};
template <> struct VecMath<__half> {
    static __device__ __forceinline__ void fma2w(float *acc, unsigned w2, float w) {
        __half2 h = *reinterpret_cast<__half2 *>(&w2);
        float2 f = __half22float2(h);
        ffma2(acc[0], acc[1], f.x, f.y, w);
    }
    static __device__ __forceinline__ void fma(float *acc, const uint4 &v, float w) {
        fma2w(acc + 0, v.x, w);
        fma2w(acc + 2, v.y, w);
        fma2w(acc + 4, v.z, w);
        fma2w(acc + 6, v.w, w);
    }
    static __device__ __forceinline__ unsigned pk(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<unsigned *>(&h);
    }
    static __device__ __forceinline__ uint4 pack(const float *a) {
        return make_uint4(pk(a[0], a[1]), pk(a[2], a[3]), pk(a[4], a[5]), pk(a[6], a[7]));
    }
};

// acc[0..8) += w * v with v eight 16-bit values and w rounded once to the
// same 16-bit type: a mixed-precision fma (16-bit multiplicands, exact product,
// fp32 accumulation and rounding), per element.
template <typename T> struct VecMathMixed;
template <> struct VecMathMixed<float> {
    static __device__ __forceinline__ void fma(float *acc, const uint4 &v, float w) {
        VecMath<float>::fma(acc, v, w);
    }
    static __device__ __forceinline__ void fma_bits(float *, const uint4 &, unsigned short) {}
};
__device__ __forceinline__ unsigned short bf16_bits(float w) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(w));
}
__device__ __forceinline__ unsigned short f16_bits(float w) {
    return __half_as_ushort(__float2half_rn(w));
}
// Two fp32 values rounded to the 16-bit type T, packed (lo in bits 0-15).
template <typename T> __device__ __forceinline__ unsigned pack2_bits(float lo, float hi);
template <> __device__ __forceinline__ unsigned pack2_bits<__nv_bfloat16>(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const unsigned *>(&h);
}
template <> __device__ __forceinline__ unsigned pack2_bits<__half>(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const unsigned *>(&h);
}
template <> __device__ __forceinline__ unsigned pack2_bits<float>(float, float) { return 0u; }
#define DCN4_MIXED_FMA(TY, CONV)                                                              \
    static __device__ __forceinline__ void fma(float *acc, const uint4 &v, float w) {        \
        fma_bits(acc, v, CONV(w));                                                            \
    }                                                                                         \
    /* the weight already rounded to the 16-bit type (its bits) */                            \
    static __device__ __forceinline__ void fma_bits(float *acc, const uint4 &v,               \
                                                    unsigned short cw) {                      \
        const unsigned wd[4] = {v.x, v.y, v.z, v.w};                                          \
        _Pragma("unroll") for (int e = 0; e < 4; ++e) {                                       \
            const unsigned short lo = (unsigned short)(wd[e] & 0xffffu);                      \
            const unsigned short hi = (unsigned short)(wd[e] >> 16);                          \
            asm("fma.rn.f32." TY " %0, %1, %2, %0;" : "+f"(acc[2 * e]) : "h"(lo), "h"(cw));   \
            asm("fma.rn.f32." TY " %0, %1, %2, %0;" : "+f"(acc[2 * e + 1]) : "h"(hi), "h"(cw)); \
        }                                                                                     \
    }
template <> struct VecMathMixed<__nv_bfloat16> { DCN4_MIXED_FMA("bf16", bf16_bits) };
template <> struct VecMathMixed<__half> { DCN4_MIXED_FMA("f16", f16_bits) };
#undef DCN4_MIXED_FMA

// acc[0..8) += w00*q00 + w01*q01 + w10*q10 + w11*q11 over eight 16-bit
// channels, the four-corner blend formed in packed 16-bit arithmetic (each
// weight rounded to T, each fused multiply-add rounded to T: the pages'
// half-precision kernel arithmetic) and added to the fp32 accumulators.
template <typename T> struct VecMathPacked;
template <> struct VecMathPacked<float> {
    static __device__ __forceinline__ void blend4(float *acc, const uint4 &q00, const uint4 &q01,
                                                  const uint4 &q10, const uint4 &q11, float w00,
                                                  float w01, float w10, float w11) {
        VecMath<float>::fma(acc, q00, w00);
        VecMath<float>::fma(acc, q01, w01);
        VecMath<float>::fma(acc, q10, w10);
        VecMath<float>::fma(acc, q11, w11);
    }
};
#define DCN4_PACKED_BLEND(T2, CVTW, TOF2)                                                        \
    static __device__ __forceinline__ void blend4(float *acc, const uint4 &q00, const uint4 &q01, \
                                                  const uint4 &q10, const uint4 &q11, float w00,  \
                                                  float w01, float w10, float w11) {              \
        const T2 a = CVTW(w00), b = CVTW(w01), c = CVTW(w10), d = CVTW(w11);                   \
        const unsigned x0[4] = {q00.x, q00.y, q00.z, q00.w}, x1[4] = {q01.x, q01.y, q01.z, q01.w}; \
        const unsigned x2[4] = {q10.x, q10.y, q10.z, q10.w}, x3[4] = {q11.x, q11.y, q11.z, q11.w}; \
        _Pragma("unroll") for (int e = 0; e < 4; ++e) {                                          \
            T2 r = __hmul2(*reinterpret_cast<const T2 *>(&x0[e]), a);                             \
            r = __hfma2(*reinterpret_cast<const T2 *>(&x1[e]), b, r);                             \
            r = __hfma2(*reinterpret_cast<const T2 *>(&x2[e]), c, r);                             \
            r = __hfma2(*reinterpret_cast<const T2 *>(&x3[e]), d, r);                             \
            const float2 f = TOF2(r);                                                            \
            const float2 s = __fadd2_rn(make_float2(acc[2 * e], acc[2 * e + 1]), f);              \
            acc[2 * e] = s.x;                                                                    \
            acc[2 * e + 1] = s.y;                                                                \
        }                                                                                        \
    }
template <> struct VecMathPacked<__nv_bfloat16> {
    DCN4_PACKED_BLEND(__nv_bfloat162, __float2bfloat162_rn, __bfloat1622float2)
};
template <> struct VecMathPacked<__half> { DCN4_PACKED_BLEND(__half2, __float2half2_rn, __half22float2) };
#undef DCN4_PACKED_BLEND

// ---- shared memory / async-copy primitives --------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- bounds-checked build (compiled with -DDCN4_CHECKED) -------------------
// Every shared- and global-memory access of the kernels is guarded by
// DCN4_SMEM_OK(p, n, base) (n bytes at p inside the CTA's dynamic shared
// memory, which starts at base) or DCN4_GMEM_OK(p, n, base, bytes) (n bytes
// at p inside the `bytes`-byte global tensor at base), or by DCN4_CHECK(cond)
// for an index bound. In a checked build a
// failing guard sets kErrInternal in the translation unit's device error word
// (g_error_word, defined before the kernels are included) and the access is
// skipped: a load yields zero, a store or atomic does nothing, a bulk copy is
// not issued (the barrier it would complete then times out, which is also
// reported). In a normal build both guards are the constant true and vanish.
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
    uint32_t r;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
    return r;
}
__device__ __forceinline__ bool smem_in(const void *p, unsigned n, const void *base) {
    const uint32_t a = smem_u32(p), b = smem_u32(base);
    return a >= b && (unsigned long long)(a - b) + n <= dynamic_smem_bytes();
}
__device__ __forceinline__ bool smem_in_u32(uint32_t a, unsigned n, const void *base) {
    const uint32_t b = smem_u32(base);
    return a >= b && (unsigned long long)(a - b) + n <= dynamic_smem_bytes();
}
__device__ __forceinline__ bool gmem_in(const void *p, unsigned n, const void *base,
                                        unsigned long long bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
    return a >= b && (unsigned long long)(a - b) + n <= bytes;
}
__device__ __forceinline__ bool flag_internal(unsigned int *word) {
    atomicOr(word, kErrInternal);
    return false;
}
#ifdef DCN4_CHECKED
#define DCN4_CHECK(cond) ((cond) || ::dcn4::flag_internal(&g_error_word))
#define DCN4_SMEM_OK(p, n, base) \
    (::dcn4::smem_in((p), (n), (base)) || ::dcn4::flag_internal(&g_error_word))
#define DCN4_SMEM_OK_U32(a, n, base) \
    (::dcn4::smem_in_u32((a), (n), (base)) || ::dcn4::flag_internal(&g_error_word))
#define DCN4_GMEM_OK(p, n, base, bytes) \
    (::dcn4::gmem_in((p), (n), (base), (bytes)) || ::dcn4::flag_internal(&g_error_word))
#else
#define DCN4_CHECK(cond) true
#define DCN4_SMEM_OK(p, n, base) true
#define DCN4_SMEM_OK_U32(a, n, base) true
#define DCN4_GMEM_OK(p, n, base, bytes) true
#endif

// Guarded 16-byte loads (zero when the guard fails).
#define DCN4_LDS16(p, base) \
    (DCN4_SMEM_OK((p), 16, (base)) ? *reinterpret_cast<const uint4 *>(p) : make_uint4(0u, 0u, 0u, 0u))
#define DCN4_LDG16(p, base, bytes)                                                   \
    (DCN4_GMEM_OK((p), 16, (base), (bytes)) ? __ldg(reinterpret_cast<const uint4 *>(p)) \
                                            : make_uint4(0u, 0u, 0u, 0u))

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of the barrier for at most `limit_ns`.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// 4-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// TMA tile store shared -> global of a 4-D box (coordinates >= 0; elements
// past the tensor's extent are not written); one bulk group per call.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Plain (untiled) bulk copy global -> shared; 16-byte aligned addresses and size.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

}  // namespace dcn4
