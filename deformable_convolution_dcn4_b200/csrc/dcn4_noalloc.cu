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
// cudaGetSymbolAddress while that device is current and caches it.
#include <mutex>

#include "dcn4.h"
#include "dcn4_launch.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_backward_scratch[kScratchBytes];

// Device address of g_backward_scratch on the current device (looked up once
// per device); nullptr when the lookup fails.
float *scratch_on_current_device() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_backward_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
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
