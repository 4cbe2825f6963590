// dcn4_launch.h -- host-side launch interface between the C ABI (dcn4_api.cu)
// and the kernel translation units (dcn4_kernels*.cu).
#pragma once

#include "dcn4_common.cuh"

namespace dcn4 {

enum class Dtype { F32 = 0, BF16 = 1, F16 = 2 };

inline int elem_bytes(Dtype t) { return t == Dtype::F32 ? 4 : 2; }

struct FwdLaunch {
    Geometry geo;
    Dtype dtype;
    bool msdcn;
    const void *in;
    const void *ow;   // offset_weight (DCNv4) or dir_weight (MSDCN)
    void *out;
    const MsdcnParams *ms;  // MSDCN only
    bool halo;              // use the shared-memory halo kernel
    bool vec;               // otherwise the vectorised global-memory kernel (else scalar)
    int mathv;              // 0 fp32 weights, 1 mixed-precision fma, 2 packed 16-bit blend
    HaloPlan plan;
    const CUtensorMap *tmap;
    const CUtensorMap *tmap_ow;  // records, when plan.rec_tma
    unsigned long long ow_bytes;
    void *ws;         // scratch for deferred escapes (16-byte aligned), or nullptr
    size_t ws_bytes;
    cudaStream_t stream;
};

// Scratch the staged forward can use for deferred escapes: entries of
// escape_entry_bytes(D, eb) for a quarter of the (pixel, group) pairs plus
// one per CTA, for up to `ctas` CTAs (eb: bytes per element).
size_t escape_entry_bytes(int D, int eb);
size_t forward_escape_bytes(long long npairs, int D, int eb, int ctas);

struct BwdLaunch {
    Geometry geo;
    Dtype dtype;
    const void *in;
    const void *ow;
    const void *gout;
    void *gin;     // element type
    void *gow;     // element type
    float *acc;    // fp32 accumulation buffer for grad_input (== gin for fp32)
    bool halo;     // use the shared-memory halo kernel
    bool vec;      // otherwise the vectorised global-memory kernel (else scalar)
    bool mixed;    // 16-bit weights with mixed-precision fma (bf16/fp16 grad_input)
    bool acc16;    // staged 16-bit kernel adds CTA partials into grad_input (no workspace)
    HaloPlan plan;
    BwdLayout layout;
    const CUtensorMap *tmap_in;
    const CUtensorMap *tmap_go;
    const CUtensorMap *tmap_ow;  // records, when plan.rec_tma
    unsigned long long ow_bytes;
    cudaStream_t stream;
    bool msdcn;             // FlowDCN multi-scale variant: ow holds (dir_x, dir_y, m)
    const MsdcnParams *ms;  // MSDCN only
    void *graw;             // MSDCN only: grad of scale_raw [N][Ho][Wo][G], element type
};

// Offset/weight producer (depthwise 3x3 + merged linear) of one call.
struct ProducerLaunch {
    ProducerGeo pg;
    Dtype dtype;
    const void *x, *dw_w, *dw_b, *lin_w, *lin_b;
    void *out;
    bool tc;    // tensor-core kernel over pixel ranges (16-bit data), else the generic kernel
    bool tc2d;  // 2-D tiled tensor-core kernel (takes precedence over tc)
    ProducerTcLayout lay;      // tc only
    ProducerTc2dLayout lay2;   // tc2d only
    const CUtensorMap *tmap_x;    // tc2d: x neighbourhoods of the tiles
    const CUtensorMap *tmap_out;  // tc2d: the tiles' output rows
    cudaStream_t stream;
};

// The fused producer + forward kernel of one call.
struct FusedLaunch {
    Geometry geo;
    Dtype dtype;  // BF16 or F16
    const void *in, *x, *dw_w, *dw_b, *lin_w, *lin_b;
    void *out;
    void *rec_out;  // optional copy of the records (offset_weight layout)
    bool records_only;  // the producer alone: no window, no gathers, out unused
    int mathv;      // as FwdLaunch::mathv
    HaloPlan plan;
    FusedLayout lay;
    const CUtensorMap *tmap_in;  // input windows
    const CUtensorMap *tmap_x;   // x neighbourhoods of the tiles
    cudaStream_t stream;
};

cudaError_t launch_forward(const FwdLaunch &L);
cudaError_t launch_producer(const ProducerLaunch &L);
cudaError_t launch_fused(const FusedLaunch &L);
cudaError_t launch_backward(const BwdLaunch &L);

// Launches the bounded-wait self-test kernel (see dcn4_selftest_bounded_wait).
cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream);

// Reads and clears the device error words of the current device (one per
// kernel translation unit, ORed).
cudaError_t read_clear_device_error(unsigned *bits);
cudaError_t read_clear_error_fwd(unsigned *bits);
cudaError_t read_clear_error_bwd(unsigned *bits);
cudaError_t read_clear_error_fused(unsigned *bits);

// Shared launch helpers (dcn4_kernels.cu): count one issued kernel; raise a
// kernel's dynamic shared-memory limit once per (kernel, device); a grid of
// ceil(work / block) blocks capped at 16 per SM.
void count_launch();
cudaError_t allow_smem(const void *kernel, int bytes);
int grid_for(long long work, int block);

// Kernels issued by this library so far (launched, or captured into a graph).
unsigned long long launches_issued();

// Number of SMs of the current device (cached per device).
int sm_count();
// Largest opt-in dynamic shared memory per block of the current device.
int max_smem_optin();
// Shared memory per SM of the current device.
int max_smem_per_sm();

}  // namespace dcn4
