// dcn4_noalloc.cu -- dcn4_backward_noalloc: the DCNv4 backward for callers
// that cannot allocate device memory.
//
// dcn4_backward needs an fp32 scratch buffer (N*H*W*C floats) for bf16/fp16
// and asks the caller to pass it in. Some callers cannot call cudaMalloc or
// any allocating routine: code that runs inside a host callback or a
// framework hook where allocation is forbidden, plugins whose host framework
// owns all device memory, or real-time code where cudaMalloc's implicit
// device synchronisation is not acceptable. This entry point takes the
// scratch from a fixed array in the library's own device memory instead.
//
// The array is a file-scope __device__ object of kScratchBytes (32 MiB): every
// GPU that loads the library holds it until the process exits. Host code may
// not pass the array's name to a kernel (on the host it is only a stand-in
// symbol), so the first call on each device looks up its device address with
// cudaGetSymbolAddress while that device is current and caches it. The
// address belongs to the CUDA context it was looked up in, so the cache is
// keyed by the context's unique id as well: after cudaDeviceReset, or when a
// caller makes another context current on the same device, the next call
// looks the address up again instead of using a stale one.
#include <cudaTypedefs.h>

#include <mutex>

#include "dcn4.h"
#include "dcn4_launch.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_backward_scratch[kScratchBytes];

// Unique id of the current driver context (cuCtxGetId, found through the
// runtime's driver entry-point query, so libcuda need not be linked); 0 when
// there is no current context or the query is unavailable.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_backward_scratch in the current device's current
// context, looked up once per (device, context); nullptr when the lookup
// fails.
float *scratch_on_current_device() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {nullptr};
    static unsigned long long ctx_of[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long ctx = current_context_id();
    if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
        void *p = nullptr;
        // also creates the device's primary context if none was current
        if (cudaGetSymbolAddress(&p, g_backward_scratch) != cudaSuccess || !p) return nullptr;
        addr[dev] = p;
        ctx_of[dev] = current_context_id();
    }
    return static_cast<float *>(addr[dev]);
}

}  // namespace

extern "C" DCN4_API dcn4_status dcn4_backward_noalloc(const dcn4_desc *desc, const void *input,
                                                      const void *offset_weight,
                                                      const void *grad_out, void *grad_input,
                                                      void *grad_offset_weight, void *stream) {
    size_t need = 0;
    if (dcn4_backward_workspace_size(desc, &need) != DCN4_OK) return DCN4_ERR_INVALID_ARG;
    if (need > kScratchBytes) return DCN4_ERR_WORKSPACE;
    if (need == 0)  // fp32: grad_input itself accumulates, no scratch needed
        return dcn4_backward(desc, input, offset_weight, grad_out, grad_input,
                             grad_offset_weight, nullptr, 0, stream);
    float *scratch = scratch_on_current_device();
    if (!scratch) return DCN4_ERR_CUDA;
    // dcn4_backward zeroes the part of the scratch it uses before accumulating.
    return dcn4_backward(desc, input, offset_weight, grad_out, grad_input, grad_offset_weight,
                         scratch, kScratchBytes, stream);
}
