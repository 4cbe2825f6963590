// dcn4_fused.cuh -- the DCNv4 module's offset/weight sub-network fused into
// the forward aggregation ("(论文速读）DCNv4：高效可变形卷积算子",
// "方法3. DCN模块的微设计优化": without softmax the offset and weight
// projections are one linear layer, fed by a depthwise 3x3 convolution):
//
//   h[p][c]      = dw_b[c] + sum_{i,j} dw_w[i][j][c] * x[p + (i-1, j-1)][c]
//   rec[p][g][.] = lin_b[.] + sum_c lin_w[.][c] * h[p][c]      (27 per group)
//   out[p][g*D + d] = the DCNv4 aggregation of `in` with the records rec[p][g]
//
// fused_halo_kernel: persistent, one CTA per SM, each CTA owns one slice of
// Gc groups (the grid is a multiple of the slice count, and unit u is slice
// u % slices of tile u / slices) and keeps that slice's rows of lin_w in
// shared memory. Per unit (TH x TW output pixels x Gc groups):
//   1. x's neighbourhood of the tile, (TH+2) x (TW+2) pixels x C, arrives by
//      one TMA tile load whose out-of-image zero fill is the depthwise
//      convolution's padding; the input window of the slice (as in the
//      forward halo kernel) arrives by a second one.
//   2. The warps compute h on the CUDA cores (fp32 from 16-bit products,
//      rounded to the data type, the tensor cores' operand type) into the
//      tcgen05 K-major core-matrix layout.
//   3. One thread issues C/16 tcgen05.mma (M = 128 tile pixels, N = the
//      slice's 27*Gc outputs padded to 16, fp32 accumulators in tensor
//      memory); the next unit's x load starts as h is consumed.
//   4. The warps read the accumulators back (tcgen05.ld), add the bias and
//      round to the data type straight into the record slots the gathers
//      read: the records reach global memory only when the caller asks for
//      them (rec_out, for a backward pass).
//   5. The forward halo kernel's gathers run on the staged window; the next
//      unit's window load then starts and overlaps its steps 1-4.
// Every wait is bounded; on expiry the CTA sets the error word, lets its
// copies and MMAs in flight land, frees its tensor memory and returns.
// With records_only the kernel is the offset/weight producer alone (steps
// 1-4 without the window, the records written to rec_out): the tensor-core
// producer for shapes whose whole lin_w does not fit one CTA next to x and h.
#pragma once

#include "dcn4_fwd.cuh"
#include "dcn4_producer.cuh"

namespace dcn4 {

// Unit u of the fused kernel: slice u % slices of tile u / slices (tiles in
// raster order within an image, images last).
__device__ __forceinline__ TileCoord fused_coord(int u, const Geometry &g, const HaloPlan &pl) {
    TileCoord c;
    const int sl = u % pl.slices;
    int t = u / pl.slices;
    const int tw = t % pl.tiles_w;
    t /= pl.tiles_w;
    const int th = t % pl.tiles_h;
    c.n = t / pl.tiles_h;
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

// Accumulators -> records: warp w reads tensor-memory lanes 32 (w & 3) ..
// +31 (tile pixels) and every (NW / 4)-th 32-column chunk from w >> 2 (a
// 16-column tail when NP % 32 != 0), adds the bias and rounds; pixel r's
// outputs land at the start of its slot, in the forward's record order
// (group, tap, (dx, dy, m)). The slot stride is an odd multiple of 16 bytes,
// so the 16-byte stores are free of bank conflicts.
template <typename T, int NW>
__device__ __forceinline__ void fused_epilogue(uint32_t tmem, const float *linb,
                                               unsigned char *slots, int slot_bytes, int NP,
                                               int npx, const unsigned char *sbase) {
    (void)sbase;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = 32 * (warp & 3) + lane;
    const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    auto store8 = [&](const float *v, int c0) {
        if (r >= npx) return;
        float fo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) fo[k] = v[k] + linb[c0 + k];
        unsigned char *dst = slots + (size_t)r * slot_bytes + c0 * 2;
        if (DCN4_SMEM_OK(dst, 16, sbase)) *reinterpret_cast<uint4 *>(dst) = pack8<T>(fo);
    };
    for (int c32 = warp >> 2; c32 < NP / 32; c32 += NW / 4) {
        float v[32];
        tc_ld_32(trow + c32 * 32, v);
#pragma unroll
        for (int h = 0; h < 4; ++h) store8(v + 8 * h, c32 * 32 + 8 * h);
    }
    if ((NP & 16) && (warp >> 2) == (NP / 32) % (NW / 4)) {
        float v[16];
        tc_ld_16(trow + (NP / 32) * 32, v);
        store8(v, (NP / 32) * 32);
        store8(v + 8, (NP / 32) * 32 + 8);
    }
}

template <typename T, int U, int MV, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    fused_halo_kernel(const __grid_constant__ CUtensorMap tmap_in,
                      const __grid_constant__ CUtensorMap tmap_x, Geometry g, HaloPlan pl,
                      FusedLayout L, const T *__restrict__ in, const T *__restrict__ dw_w,
                      const T *__restrict__ dw_b, const T *__restrict__ lin_w,
                      const T *__restrict__ lin_b, T *__restrict__ out,
                      T *__restrict__ rec_out, const __grid_constant__ MsdcnParams ms,
                      int records_only) {
    extern __shared__ __align__(1024) unsigned char smem[];
    constexpr int NT = NW * 32;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int C = g.C, Q = C / 8;
    const int npx = pl.TH * pl.TW;
    const int units = g.N * pl.tiles_h * pl.tiles_w * pl.slices;
    const int sl = (int)blockIdx.x % pl.slices;  // the grid is a multiple of pl.slices
    unsigned char *win = smem + L.win_off, *slots = smem + L.slots_off, *xs = smem + L.x_off;
    unsigned char *abuf = smem + L.a_off;
    T *dwt = reinterpret_cast<T *>(smem + L.dwt_off);
    float *dwb = reinterpret_cast<float *>(smem + L.dwb_off);
    float *linb = reinterpret_cast<float *>(smem + L.linb_off);
    const uint32_t x_bar = smem_u32(smem + L.bar_off), win_bar = x_bar + 8, mma_bar = x_bar + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.bar_off + 24);
    // tensor extents (bounds of the checked build; unused otherwise)
    const unsigned long long lw_b = (unsigned long long)g.G * 27 * C * 2;
    const unsigned long long ow_b = (unsigned long long)g.N * g.Ho * g.Wo * g.G * 27 * 2;
    (void)lw_b, (void)ow_b;

    // resident operands: the slice's lin_w rows in core-matrix layout (rows
    // >= JS zero), the depthwise taps, both biases in fp32; rows of h past
    // the tile's pixels zero for good
    for (int i = tid; i < L.NP * Q; i += NT) {
        const int n = i / Q, q = i - n * Q;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < L.JS) v = DCN4_LDG16(lin_w + (size_t)(sl * L.JS + n) * C + q * 8, lin_w, lw_b);
        if (DCN4_SMEM_OK(smem + L.b_off + core_off(n, q, C), 16, smem))
            *reinterpret_cast<uint4 *>(smem + L.b_off + core_off(n, q, C)) = v;
    }
    for (int i = npx * Q + tid; i < 128 * Q; i += NT) {
        const int r = i / Q, q = i - r * Q;
        if (DCN4_SMEM_OK(abuf + core_off(r, q, C), 16, smem))
            *reinterpret_cast<uint4 *>(abuf + core_off(r, q, C)) = make_uint4(0, 0, 0, 0);
    }
    if (DCN4_SMEM_OK(dwt, 9 * C * 2, smem) && DCN4_SMEM_OK(dwb, C * 4, smem) &&
        DCN4_SMEM_OK(linb, L.NP * 4, smem)) {
        for (int i = tid; i < 9 * C; i += NT) dwt[i] = dw_w[i];
        for (int i = tid; i < C; i += NT) dwb[i] = Elem<T>::to_f(dw_b[i]);
        for (int i = tid; i < L.NP; i += NT)
            linb[i] = i < L.JS ? Elem<T>::to_f(lin_b[sl * L.JS + i]) : 0.f;
    }
    if (tid == 0) {
        mbar_init(x_bar, 1);
        mbar_init(win_bar, 1);
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
    const uint32_t idesc = umma_idesc_f16(std::is_same<T, __nv_bfloat16>::value, 128, L.NP);
    const uint32_t a_base = smem_u32(abuf), b_base = smem_u32(smem + L.b_off);

    // thread 32 issues the x loads, thread 0 the window loads and the MMAs
    // (so the next x load and the MMAs go out side by side); each counts its
    // own, so that a CTA leaving on an expired wait can let the outstanding
    // ones land first
    constexpr int kXThread = 32;
    int x_issued = 0, x_done = 0, win_issued = 0, win_done = 0, mma_issued = 0, mma_done = 0;
    auto issue_x = [&](const TileCoord &tc) {
        fence_async_smem();  // the generic reads of the buffer come first
        mbar_arrive_expect_tx(x_bar, (uint32_t)L.x_bytes);
        if (DCN4_SMEM_OK(xs, (unsigned)L.x_bytes, smem))
            tma_load_4d(smem_u32(xs), &tmap_x, 0, tc.wo0 - 1, tc.ho0 - 1, tc.n, x_bar);
        ++x_issued;
    };
    auto issue_win = [&](const TileCoord &tc) {
        stage_window(tc, &tmap_in, g, pl, Elem<T>::kBytes, win, win_bar, smem);
        ++win_issued;
    };
    bool ok = true;
    // unit k (index u): its depthwise outputs into A, then (thread 0) the x
    // load of unit k+1 into the consumed buffer and unit k's MMA, which runs
    // on the tensor cores while the warps go on; false on an expired wait
    // (every thread gets the same answer)
    auto produce = [&](int k, int u) -> bool {
        if (!mbar_wait_bounded(x_bar, (uint32_t)k & 1u, kWaitLimitNs)) ok = false;
        else if (tid == kXThread) ++x_done;
        if (__syncthreads_or(!ok)) return false;
        depthwise_tile<T, NW, 4>(xs, abuf, dwt, dwb, C, pl.TH, pl.TW, pl.lgTW, smem);
        fence_async_smem();
        __syncthreads();
        if (tid == kXThread && u + (int)gridDim.x < units)
            issue_x(fused_coord(u + gridDim.x, g, pl));
        if (tid == 0) {
            tc_fence_after();
            for (int kk = 0; kk < C / 16; ++kk)
                tc_mma_f16(tmem, umma_desc_kmajor(a_base + kk * 256, 128, C * 16),
                           umma_desc_kmajor(b_base + kk * 256, 128, C * 16), idesc, kk > 0);
            tc_commit(mma_bar);
            ++mma_issued;
        }
        return true;
    };
    // unit k's records: accumulators -> slots (and, when asked for, to
    // rec_out: a slice's Gc*27 values of a pixel start at an even element,
    // so 4-byte words)
    auto finish = [&](int k, const TileCoord &tc) -> bool {
        if (!mbar_wait_bounded(mma_bar, (uint32_t)k & 1u, kWaitLimitNs)) ok = false;
        else if (tid == 0) ++mma_done;
        if (__syncthreads_or(!ok)) return false;
        tc_fence_after();
        fused_epilogue<T, NW>(tmem, linb, slots, pl.slot_bytes, L.NP, npx, smem);
        tc_fence_before();
        __syncthreads();
        if (rec_out != nullptr) {
            const int wpp = L.JS / 2;  // words per pixel of the slice
            for (int i = tid; i < npx * wpp; i += NT) {
                const int r = i / wpp, w = i - r * wpp;
                const int ty = r >> pl.lgTW, tx = r & (pl.TW - 1);
                if (ty >= tc.th_eff || tx >= tc.tw_eff) continue;
                const unsigned long long gp = tc.gp0 + (unsigned long long)ty * g.Wo + tx;
                uint32_t *dst = reinterpret_cast<uint32_t *>(rec_out) +
                                (gp * g.G + tc.g0) * 27 / 2 + w;
                const unsigned char *src = slots + (size_t)r * pl.slot_bytes + 4 * w;
                if (DCN4_GMEM_OK(dst, 4, rec_out, ow_b) && DCN4_SMEM_OK(src, 4, smem))
                    *dst = *reinterpret_cast<const uint32_t *>(src);
            }
        }
        return true;
    };

    // Per unit: produce (x wait, depthwise, MMA issue, next x load), finish
    // (MMA wait, records), the gathers, then the next unit's window load.
    // (Issuing unit k+1's MMA before unit k's gathers, so that it runs under
    // them, measured slower on the InternImage stage: 244 against 231 us.)
    if ((int)blockIdx.x < units) {
        const TileCoord t0 = fused_coord(blockIdx.x, g, pl);
        if (tid == kXThread) issue_x(t0);
        if (tid == 0 && !records_only) issue_win(t0);
        int k = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++k) {
            const TileCoord tc = fused_coord(u, g, pl);
            const int un = u + gridDim.x;
            if (!produce(k, u) || !finish(k, tc)) break;
            if (records_only) continue;  // the producer alone: records to rec_out
            if (!mbar_wait_bounded(win_bar, (uint32_t)k & 1u, kWaitLimitNs)) ok = false;
            else if (tid == 0) ++win_done;
            if (__syncthreads_or(!ok)) break;
            compute_tile<T, U, false, MV, 1>(tc, g, pl, in, out, ms, win, slots, tid, NT, smem);
            __syncthreads();
            if (tid == 0 && un < units) issue_win(fused_coord(un, g, pl));
        }
    }

    // at most one copy of each kind and one MMA batch are outstanding
    if (tid == kXThread && !ok && x_issued > x_done)
        mbar_wait_bounded(x_bar, (uint32_t)(x_issued - 1) & 1u, kWaitLimitNs);
    if (tid == 0 && !ok) {
        atomicOr(&g_error_word, kErrTimeout);
        if (win_issued > win_done)
            mbar_wait_bounded(win_bar, (uint32_t)(win_issued - 1) & 1u, kWaitLimitNs);
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

}  // namespace dcn4
