/*
 * dcn4.h -- C ABI of the B200 (sm_100a) DCNv4 deformable spatial aggregation
 * library (libdcn4.so).
 *
 * The operation (DCNv4, CVPR 2024; as summarised in "(论文速读）DCNv4：高效可变形
 * 卷积算子", sections "移除Softmax归一化" and "方法1. 消除冗余工作负载", and in
 * "NeurIPS'24 | FlowDCN：基于可变形卷积的任意分辨率图像生成模型", section
 * "2.2 DCN结构简介"): for every output pixel p0 = (ho, wo), group g and kernel
 * tap k = (i, j), sample the channel-last input by bilinear interpolation at
 *
 *     x = (wo*stride_w - pad_w + j*dil_w) + dx * offset_scale
 *     y = (ho*stride_h - pad_h + i*dil_h) + dy * offset_scale
 *
 * (in-image corners only; a sample outside (-1, W) x (-1, H) adds nothing),
 * multiply the sample by the unnormalised weight m (no softmax), sum over the
 * taps and write the D = C/G channels of group g into their slot of the
 * C-vector (the groups are concatenated).
 *
 * Tensors (all dense, contiguous, channel-last, one element type per call):
 *   input          [N][H][W][C]
 *   offset_weight  [N][Ho][Wo][G][kh*kw][3]   triples (dx along W, dy along H, m),
 *                                             tap k = i*kw + j, i along H
 *   output         [N][Ho][Wo][C]
 *   Ho = (H + 2*pad_h - dil_h*(kh-1) - 1) / stride_h + 1, likewise Wo.
 *
 * Arithmetic: sample positions are formed in fp32 with the product
 * dx*offset_scale and the sum each rounded to nearest (no fused multiply-add),
 * so corner indices match a CPU evaluation of the same formula bit for bit;
 * interpolation weights and accumulation are fp32; results are rounded once
 * to the element type.
 *
 * Conventions for every entry point:
 *   - Device pointers are owned by the caller; the library allocates no memory
 *     and keeps no per-call state. Exceptions: a device error word (see
 *     dcn4_last_device_error), a launch counter (dcn4_kernel_launches), and
 *     the fixed 32 MiB scratch array of dcn4_backward_noalloc together with
 *     its per-(device, context) address cache (see that entry point).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Calls only enqueue work; they never synchronise the device.
 *   - Outputs are overwritten, never accumulated into.
 *   - Argument errors are reported synchronously before anything is
 *     launched; launch failures come back as DCN4_ERR_CUDA.
 *   - Pointers that are not 16-byte aligned, or channel counts whose group
 *     slice is not a multiple of 16 bytes, are legal: such calls take the
 *     generic (slower) kernels.
 */
#ifndef DCN4_H
#define DCN4_H

#include <stddef.h>

#if defined(DCN4_BUILDING_LIBRARY) && defined(__GNUC__)
#define DCN4_API __attribute__((visibility("default")))
#else
#define DCN4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DCN4_OK = 0,
    DCN4_ERR_INVALID_ARG = 1,  /* malformed descriptor or null pointer        */
    DCN4_ERR_UNSUPPORTED = 2,  /* well formed but outside what is implemented */
    DCN4_ERR_WORKSPACE = 3,    /* workspace missing or too small              */
    DCN4_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed        */
    DCN4_ERR_TIMEOUT = 5,      /* a device-side bounded wait expired          */
    DCN4_ERR_INTERNAL = 6      /* a device-side consistency check failed      */
} dcn4_status;

typedef enum { DCN4_F32 = 0, DCN4_BF16 = 1, DCN4_F16 = 2 } dcn4_dtype;

/* Kernel selection. AUTO picks the staged (shared-memory halo) kernel when
 * the call qualifies and a global-memory kernel otherwise: the vectorised one
 * (16-byte vector loads, several threads per (pixel, group)) when a group's
 * channels are whole 16-byte vectors (backward: a power-of-two count of them,
 * at most 16) and the tensors are 16-byte aligned, else the scalar one.
 * GENERIC forces the scalar global-memory kernel, VECTOR the vectorised one
 * and HALO the staged one (a forced variant the call does not qualify for
 * returns DCN4_ERR_UNSUPPORTED). */
typedef enum {
    DCN4_ALGO_AUTO = 0,
    DCN4_ALGO_GENERIC = 1,
    DCN4_ALGO_HALO = 2,
    DCN4_ALGO_VECTOR = 3
} dcn4_algo;

/* Multiply precision of the bilinear weights in the bf16/fp16 halo kernels
 * (fp32 calls and the generic kernels always use fp32).
 *   F32      bilinear weights in fp32; every product and sum in fp32.
 *   MIXED16  each weight is rounded once to the input's 16-bit type and the
 *            sm_100 mixed-precision fma multiplies it with the 16-bit data
 *            (exact 16x16-bit product, fp32 accumulation). The extra error is
 *            one 16-bit rounding of each weight (relative 2^-9 for bf16,
 *            2^-12 for fp16), the size of the data's own quantisation; sums
 *            stay fp32.
 *   PACKED16 forward only (the backward runs as MIXED16): the four-corner
 *            blend of each tap is formed in packed 16-bit arithmetic
 *            (bf16x2/f16x2 fused multiply-adds, each rounded to the data type,
 *            as in the half-precision kernel of "(论文速读）DCNv4：高效可变形卷积算子",
 *            "方法2") and added to fp32 accumulators over the taps. About
 *            twice the error of MIXED16 (rms relative ~3e-3 for bf16,
 *            ~4e-4 for fp16, against ~1.7e-3 / ~2e-4 for the rounding of
 *            the output itself), for fewer instructions per tap.
 *   ACC16    bf16/fp16 backward only (the forward runs as MIXED16): as
 *            MIXED16, but the staged kernel adds each CTA's fp32 partial sum
 *            of grad_input straight into the 16-bit grad_input with packed
 *            16-bit atomic adds (one rounding per contributing CTA, up to
 *            ~6 per element, plus one per sample that leaves the staged
 *            window), skipping the fp32 workspace and its zero and convert
 *            passes. Faster, not fp32-accumulated across CTAs.
 *   DEFAULT  MIXED16 for bf16/fp16 data, F32 for fp32 data.
 * In every mode except ACC16, grad_input is accumulated in fp32 across the
 * whole call (the workspace for bf16/fp16) and rounded once at the end.
 * Dot products of two stored tensors (the backward's <grad_out, input>) are
 * exact products of the stored values summed in fp32 in every mode. */
typedef enum {
    DCN4_MATH_DEFAULT = 0,
    DCN4_MATH_F32 = 1,
    DCN4_MATH_MIXED16 = 2,
    DCN4_MATH_PACKED16 = 3,
    DCN4_MATH_ACC16 = 4
} dcn4_math;

/* Aggregation weights ("(论文速读）DCNv4：高效可变形卷积算子", "移除Softmax归一化"):
 *   PLAIN    DCNv4: m is used as given (unbounded, no normalisation).
 *   SOFTMAX  DCNv3 compatibility: the K values m of one (pixel, group) are
 *            replaced by softmax(m) over the taps (largest subtracted first,
 *            fp32 expf); the backward returns the gradient with respect to
 *            the logits m. DCNv4 calls only (MSDCN returns UNSUPPORTED). */
typedef enum { DCN4_WEIGHTS_PLAIN = 0, DCN4_WEIGHTS_SOFTMAX = 1 } dcn4_weights;

/* Where the MSDCN scale acts ("NeurIPS'24 | FlowDCN", "3.1"; the page's
 * formula is missing and both readings fit its text):
 *   SCALE_OFFSET    the offset is s * dir: sample = p0 + p_k + s*dir*os.
 *   SCALE_DILATION  the scale stretches the kernel grid too:
 *                   sample = c + s * (p_k + dir*os), c the centre of the
 *                   kh x kw window, p_k the tap's grid offset from it
 *                   ((j - (kw-1)/2) * dil_w, (i - (kh-1)/2) * dil_h);
 *                   every product and sum rounded to fp32 in that order.
 * DCNv4 calls ignore this field. */
typedef enum { DCN4_MSDCN_SCALE_OFFSET = 0, DCN4_MSDCN_SCALE_DILATION = 1 } dcn4_msdcn_mode;

/* The whole configuration of one call. Limits: all sizes positive, C % G == 0,
 * G <= 1024, 1 <= kh*kw <= 64, strides and dilations >= 1, pads >= 0, every
 * tensor below 2^31 elements, Ho and Wo positive. */
typedef struct {
    int N, H, W, C, G;
    int kh, kw;
    int stride_h, stride_w;
    int pad_h, pad_w;
    int dil_h, dil_w;
    float offset_scale;
    dcn4_dtype dtype;
    dcn4_algo algo;
    dcn4_math math;
    dcn4_weights weights;
    dcn4_msdcn_mode msdcn_mode;
} dcn4_desc;

/* Output size for `desc` (standard convolution arithmetic, as in
 * "CANN ops-nn 算子与 Stable Diffusion 的卷积实现", "2.1 标准卷积的数学表达").
 * Returns DCN4_ERR_INVALID_ARG for a malformed descriptor. */
DCN4_API dcn4_status dcn4_out_shape(const dcn4_desc *desc, int *Ho, int *Wo);

/* DCNv4 forward (definition above). input, offset_weight and output are
 * device pointers of desc->dtype with the shapes above; output must not
 * overlap the inputs. */
DCN4_API dcn4_status dcn4_forward(const dcn4_desc *desc, const void *input,
                         const void *offset_weight, void *output, void *stream);

/* Bytes of device scratch with which dcn4_forward_ws and msdcn_forward_ws
 * run fastest for `desc` (0 where the staged kernel cannot use any: taps
 * other than 3x3, groups other than 2 (bf16/fp16) or 4 16-byte vectors, or
 * DCN4_ALGO_GENERIC/VECTOR): 16 + 4*D bytes for a quarter of the N*Ho*Wo*G
 * (pixel, group) pairs plus one per CTA, for up to 8 CTAs per SM. */
DCN4_API dcn4_status dcn4_forward_workspace_size(const dcn4_desc *desc, size_t *bytes);

/* dcn4_forward with scratch for the staged kernel's escapes (samples outside
 * its shared-memory window; no counterpart on the pages). In place, a warp
 * waits on the global loads of any one lane's escaped tap; with scratch, a
 * (pixel, group) pair with escaped taps writes its in-window partial sums
 * (fp32) and the taps' mask to `workspace` instead of its output, and its
 * CTA, after its last tile, adds those taps with all its threads (global
 * loads, the same arithmetic in the same order) and writes the output. One
 * kernel either way; the output is bit-identical to dcn4_forward's.
 * workspace: device memory owned by the caller, 16-byte aligned, or NULL;
 * any size is accepted (none, a misaligned pointer or too little for one
 * entry per CTA: escapes are handled in place; a CTA whose share of the
 * entries fills up handles further escapes in place). Two calls must not
 * use the same workspace at the same time. */
DCN4_API dcn4_status dcn4_forward_ws(const dcn4_desc *desc, const void *input,
                                     const void *offset_weight, void *output, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* Bytes of device workspace dcn4_backward needs for `desc`: an fp32 copy of
 * grad_input for bf16/fp16 (N*H*W*C*4 bytes) and 0 for fp32. (Under
 * DCN4_MATH_ACC16 the staged bf16/fp16 kernel accumulates in grad_input
 * itself and leaves the workspace unused; every other bf16/fp16 call uses
 * it.) */
DCN4_API dcn4_status dcn4_backward_workspace_size(const dcn4_desc *desc, size_t *bytes);

/* DCNv4 backward: the derivative of the forward (the pages only say that
 * DCNv4 optimised its backward operator; FlowDCN article, "2.2" and "4.1").
 * Reads input, offset_weight and grad_out ([N][Ho][Wo][C]); writes
 *   grad_input          [N][H][W][C]     sum over samples of m*w_corner*grad_out
 *   grad_offset_weight  [N][Ho][Wo][G][kh*kw][3]
 *       (d/d dx, d/d dy, d/d m) of sum(output * grad_out).
 * At an integer sample position the derivative is that of the cell floor()
 * selects. `workspace` (>= dcn4_backward_workspace_size bytes, 16-byte
 * aligned, device memory owned by the caller) may be NULL when that size is 0.
 * grad_input sums partial results with fp32 atomic adds (in the workspace for
 * bf16/fp16, rounded once to the element type at the end), so its last bits
 * may vary from run to run; under DCN4_MATH_ACC16 the staged bf16/fp16
 * kernel adds each CTA's fp32 partial sum to grad_input with one 16-bit
 * rounding instead. */
DCN4_API dcn4_status dcn4_backward(const dcn4_desc *desc, const void *input,
                          const void *offset_weight, const void *grad_out,
                          void *grad_input, void *grad_offset_weight,
                          void *workspace, size_t workspace_bytes, void *stream);

/* MSDCN (groupwise multi-scale DCN) forward, "NeurIPS'24 | FlowDCN", section
 * "3.1 组间多尺度可变形卷积": the offset of group g, tap k at pixel p0 is
 * s_g(p0) * dir_{g,k}(p0) with
 *     s_g = min(s0[g] * softplus(scale_raw), smax),
 *     softplus(r) = max(r, 0) + log1p(exp(-|r|))       (fp32, expf/log1pf),
 * after which the sample is formed exactly as in dcn4_forward (offset_scale
 * still applies). dir_weight [N][Ho][Wo][G][kh*kw][3] holds (dir_x, dir_y, m);
 * scale_raw [N][Ho][Wo][G] (device, desc->dtype); s0_host [G] is a HOST array
 * of fp32 scale priors, copied into the launch. A NaN scale gives no
 * contribution. */
DCN4_API dcn4_status msdcn_forward(const dcn4_desc *desc, const void *input,
                          const void *dir_weight, const void *scale_raw,
                          const float *s0_host, float smax, void *output,
                          void *stream);

/* msdcn_forward with scratch for the staged kernel's escapes, as
 * dcn4_forward_ws (size from dcn4_forward_workspace_size; the output is
 * bit-identical to msdcn_forward's). */
DCN4_API dcn4_status msdcn_forward_ws(const dcn4_desc *desc, const void *input,
                                      const void *dir_weight, const void *scale_raw,
                                      const float *s0_host, float smax, void *output,
                                      void *workspace, size_t workspace_bytes, void *stream);

/* MSDCN backward: the derivative of msdcn_forward (FlowDCN article, "3.1";
 * the page prints no gradient, these follow by the chain rule). With
 * g_x, g_y the derivatives of sum(output * grad_out) with respect to the
 * sample position of tap k (computed as in dcn4_backward):
 *   grad_input        [N][H][W][C]           as in dcn4_backward
 *   grad_dir_weight   [N][Ho][Wo][G][kh*kw][3]
 *       d/d dir_x = s * offset_scale * g_x, d/d dir_y = s * offset_scale * g_y,
 *       d/d m as in dcn4_backward
 *   grad_scale_raw    [N][Ho][Wo][G]
 *       (ds/draw) * offset_scale * sum_k (g_x dir_x + g_y dir_y), where
 *       ds/draw = s0 * sigmoid(raw) while s0 * softplus(raw) <= smax and 0
 *       once the clamp is active (or raw is NaN).
 * Arguments as in msdcn_forward and dcn4_backward (grad outputs in
 * desc->dtype, device; the same workspace size, dcn4_backward_workspace_size).
 * Kernels: AUTO runs the staged shared-memory kernel of dcn4_backward (with
 * the multi-scale positions; its window is the same, so more samples take its
 * global path) when the call qualifies for it as a dcn4_backward call would
 * (3x3 taps, a group of 2 or 4 16-byte vectors, 16-byte aligned tensors), and
 * grad_input then accumulates as in dcn4_backward; otherwise grad_input
 * accumulates with fp32 atomics in the workspace (fp32 data: in grad_input)
 * from D*sizeof(T)/16 lanes per (pixel, group) with 16-byte vector loads when
 * the group is a power-of-two count of 16-byte vectors (up to 16) and the
 * tensors are 16-byte aligned, else (and under DCN4_ALGO_GENERIC) from one
 * thread per (pixel, group) with scalar atomics. DCN4_ALGO_HALO and
 * DCN4_ALGO_VECTOR demand their kernel (DCN4_ERR_UNSUPPORTED where it does not
 * apply). desc->weights must be DCN4_WEIGHTS_PLAIN. */
DCN4_API dcn4_status msdcn_backward(const dcn4_desc *desc, const void *input,
                          const void *dir_weight, const void *scale_raw,
                          const float *s0_host, float smax, const void *grad_out,
                          void *grad_input, void *grad_dir_weight, void *grad_scale_raw,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Offset/weight producer of the DCNv4 module ("(论文速读）DCNv4：高效可变形卷积算子",
 * "方法3. DCN模块的微设计优化": once softmax is removed the offset and weight
 * projections merge into one linear layer, and the sub-network in front of it
 * is a plain separable convolution: a depthwise 3x3 convolution, then that
 * linear layer, without DCNv3's LayerNorm and GELU). For every pixel p of the
 * H x W map x [N][H][W][C]:
 *   h[p][c]   = dw_bias[c] + sum_{i,j in 0..2} dw_weight[i][j][c] * x[p + (i-1, j-1)][c]
 *               (stride 1, zero outside the image)
 *   offset_weight[p][j] = lin_bias[j] + sum_c lin_weight[j][c] * h[p][c],
 *               j in [0, G*kh*kw*3),
 * i.e. offset_weight comes out as [N][H][W][G][kh*kw][3] (dx, dy, m per tap),
 * ready for dcn4_forward with the same desc. dw_weight is [3][3][C]
 * (tap-major), dw_bias [C], lin_weight [G*kh*kw*3][C] (one row per output),
 * lin_bias [G*kh*kw*3]; all are device pointers of desc->dtype. The layer
 * serves the sampling grid of `desc`, so the output grid must be the input
 * grid (Ho == H, Wo == W; else DCN4_ERR_UNSUPPORTED); stride, pad and dilation
 * matter only through that check.
 * Precision: fp32 accumulation throughout. bf16/fp16 calls round h to the data
 * type before the linear layer (the tensor cores take 16-bit operands); the
 * result is rounded once to the data type.
 * Kernels: bf16/fp16 with C % 16 == 0, G*kh*kw*3 <= 256, whole 16-byte output
 * rows ((G*kh*kw*3*2) % 16 == 0), lin_weight fitting one CTA's shared memory
 * next to x and h, and 16-byte aligned x, lin_weight and offset_weight use
 * the tensor-core (tcgen05) kernels (2-D tiles where they fit, else pixel
 * ranges). Other bf16/fp16 calls with 3x3 taps and the shapes
 * dcn4_fused_forward's kernel takes (D*2 in {32, 64} bytes, C a multiple of
 * 64, C <= 256; 16-byte aligned x and lin_weight, 4-byte aligned
 * offset_weight) run that kernel's producer steps alone: each CTA computes
 * the outputs of one slice of 128 bytes of groups on the tensor cores (the
 * depthwise pass repeated per slice). Every other call, and desc->algo ==
 * DCN4_ALGO_GENERIC, runs the CUDA-core kernel (h kept in fp32).
 * DCN4_ALGO_HALO demands a tensor-core kernel (DCN4_ERR_UNSUPPORTED where
 * none applies). */
DCN4_API dcn4_status dcn4_offset_producer(const dcn4_desc *desc, const void *x,
                                          const void *dw_weight, const void *dw_bias,
                                          const void *lin_weight, const void *lin_bias,
                                          void *offset_weight, void *stream);

/* Scratch bytes dcn4_fused_forward may need for this desc: 0 when the call
 * runs the fused kernel (its shape and desc->algo; it may still need the
 * scratch when a pointer is not aligned, see below), else the size of the
 * offset_weight tensor the two-kernel chain passes through,
 * N*Ho*Wo*G*kh*kw*3 elements of desc->dtype rounded up to 16 bytes (none is
 * needed when the call passes offset_weight_out), plus
 * dcn4_forward_workspace_size bytes for the forward's escapes (optional:
 * the chain's forward uses what the records leave over, see
 * dcn4_forward_ws). With DCN4_ALGO_AUTO that includes the shapes on
 * which the chain is the faster path (see dcn4_fused_forward); a call given
 * no scratch there runs the fused kernel instead. */
DCN4_API dcn4_status dcn4_fused_forward_workspace_size(const dcn4_desc *desc, size_t *bytes);

/* The DCNv4 module's aggregation with its offset/weight sub-network in front
 * ("(论文速读）DCNv4：高效可变形卷积算子", "方法3. DCN模块的微设计优化": the offset
 * and weight projections become one linear layer after a depthwise 3x3
 * convolution): output = dcn4_forward(input, dcn4_offset_producer(x, ...))
 * with the same desc, without the N*Ho*Wo*G*kh*kw*3 offset_weight tensor
 * going through global memory when the fused kernel runs.
 *   input [N][H][W][C] (the sampled map), x [N][H][W][C] (the map the
 *   offsets and weights are computed from), dw_weight [3][3][C], dw_bias [C],
 *   lin_weight [G*kh*kw*3][C], lin_bias [G*kh*kw*3], output [N][Ho][Wo][C]:
 *   device pointers of desc->dtype, owned by the caller. As for the producer,
 *   Ho == H and Wo == W (else DCN4_ERR_UNSUPPORTED).
 *   offset_weight_out: NULL, or [N][Ho][Wo][G][kh*kw][3] of desc->dtype, which
 *   then receives the records the aggregation used (what dcn4_backward takes
 *   as offset_weight in a training step; one extra write of that tensor).
 * Result: what the two calls give, records rounded to the data type in
 * between, fp32 accumulation in both steps.
 * Kernels: bf16/fp16 with a 3x3 kernel, D*2 in {32, 64} bytes, G a multiple
 * of 128 / (D*2) (hence C a multiple of 64), C <= 256, 16-byte aligned
 * input, x, lin_weight and output, a 4-byte aligned offset_weight_out,
 * desc->weights either mode and a tile that fits shared memory run one
 * persistent tcgen05 kernel per call: each CTA owns an output tile x a slice
 * of groups, loads the tile's x neighbourhood by TMA, computes the depthwise
 * outputs on the CUDA cores, the slice's rows of the linear layer on the
 * tensor cores (accumulators in tensor memory), and writes the records
 * straight into the shared-memory slots the gathers read. Every other call
 * (and DCN4_ALGO_GENERIC or DCN4_ALGO_VECTOR, which select the forward kernel
 * of the second step) runs dcn4_offset_producer into offset_weight_out, or
 * when that is NULL into `workspace` (at least
 * N*Ho*Wo*G*kh*kw*3*sizeof(element) bytes, else DCN4_ERR_WORKSPACE before any
 * launch; 16-byte aligned to take the tensor-core producer and the staged
 * forward), and then dcn4_forward on it. The chain's records are the
 * tensor-core producers' where one applies and the CUDA-core producer's
 * (h kept in fp32) otherwise, so on shapes no tensor-core producer takes the
 * chain and the fused kernel may round a record differently.
 * DCN4_ALGO_AUTO also takes the chain on a fused-kernel shape where the
 * chain is faster, when it has 16-byte aligned room for the records
 * (offset_weight_out, or a large enough workspace): where the groups span
 * two or more slices (every slice's CTA then repeats the depthwise pass) and
 * the tensor-core producer takes the shape in one 2-D tiled pass (at most 256
 * outputs per pixel in whole 16-byte rows, C and lin_weight fitting shared
 * memory) -- the InternImage stage, C128 G8, is one -- and where they span
 * four slices or more (C256 G16, C256 G8), whose producer runs this kernel's
 * producer steps alone. Given no room it runs the fused kernel.
 * DCN4_ALGO_HALO demands the fused kernel (DCN4_ERR_UNSUPPORTED where it does
 * not apply). */
DCN4_API dcn4_status dcn4_fused_forward(const dcn4_desc *desc, const void *input, const void *x,
                                        const void *dw_weight, const void *dw_bias,
                                        const void *lin_weight, const void *lin_bias,
                                        void *output, void *offset_weight_out,
                                        void *workspace, size_t workspace_bytes, void *stream);

/* dcn4_backward for callers that cannot allocate device memory. The paper
 * has no counterpart; this is a deployment convenience. dcn4_backward needs
 * an fp32 scratch buffer for bf16/fp16 that the caller must allocate; callers
 * that may not call cudaMalloc (host callbacks and framework hooks that forbid
 * allocation, plugins whose framework owns all device memory, real-time code
 * that cannot accept cudaMalloc's implicit synchronisation) use this entry
 * point instead, which takes the scratch from a fixed 32 MiB array inside the
 * library (held on every GPU that loads the library until the process exits)
 * and allocates nothing.
 *   - Limit: dcn4_backward_workspace_size(desc) must be <= 32 MiB
 *     (N*H*W*C <= 8,388,608 for bf16/fp16); larger calls return
 *     DCN4_ERR_WORKSPACE without launching. The limit applies to every
 *     bf16/fp16 call, also to those whose kernels end up not touching the
 *     scratch. fp32 calls need no scratch and have no limit.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream
 *     capture. The address is cached per (device, CUDA context): a call made
 *     under another context (after cudaDeviceReset, or a context the caller
 *     made current through the driver API) looks it up again.
 *   - All calls on a device share the one array; each call zeroes the part it
 *     uses first, but calls that overlap on the GPU (different streams, or
 *     several host threads) race on it and give wrong results.
 * Arguments, outputs and errors are otherwise those of dcn4_backward. */
DCN4_API dcn4_status dcn4_backward_noalloc(const dcn4_desc *desc, const void *input,
                                           const void *offset_weight, const void *grad_out,
                                           void *grad_input, void *grad_offset_weight,
                                           void *stream);

/* Diagnostic for failure detection (no counterpart on the pages): launches one
 * CTA whose mbarrier expects 16 bytes that no copy ever delivers, so its
 * bounded wait gives up after `timeout_us` microseconds (clamped to
 * 1..2,000,000) and sets the DCN4_ERR_TIMEOUT bit of the device error word,
 * exactly as a stalled copy in the real kernels would. Nothing faults or
 * hangs; read the result with dcn4_last_device_error after the stream has
 * drained. */
DCN4_API dcn4_status dcn4_selftest_bounded_wait(unsigned int timeout_us, void *stream);

/* Human-readable name of a status code (static storage). */
DCN4_API const char *dcn4_status_string(dcn4_status status);

/* Reads and clears the device error word that kernels set when a bounded wait
 * expires (DCN4_ERR_TIMEOUT) or a consistency check fails
 * (DCN4_ERR_INTERNAL). *code receives the raw bit set (0 = none). This call
 * synchronises the current device. Returns DCN4_OK when the word was clear,
 * otherwise the status the bits map to. */
DCN4_API dcn4_status dcn4_last_device_error(unsigned int *code);

/* Number of kernels this library has issued in this process, summed over
 * devices and threads: every kernel launch, including launches recorded into
 * a CUDA graph under stream capture (a graph replays them without passing
 * through the library, so a caller counts replays itself). The pages define
 * no such call; it lets a benchmark state how many of the library's kernels
 * ran. *count receives the value. Never fails except on a null pointer
 * (DCN4_ERR_INVALID_ARG). */
DCN4_API dcn4_status dcn4_kernel_launches(unsigned long long *count);

#ifdef __cplusplus
}
#endif

#endif /* DCN4_H */
