// qmv_qvm_noalloc.cu -- qmv_qvm_affine_noalloc: the qvm call for callers that
// cannot allocate device memory, with its K-split scratch in a fixed array
// that the library itself holds.
//
// The pages have no counterpart: this entry point exists for library users.
// Some callers must not allocate device memory at all.  Examples are a plugin
// whose host framework owns every device byte through its own pool and
// forbids driver allocations, and a latency-critical decode loop that cannot
// afford the device synchronization a cudaMalloc / cudaFree may imply.  Such a
// caller cannot provide qmv_qvm_affine's workspace, and without one qvm keeps
// each 1024-column tile in a single block (few blocks unless N is large).
// This entry point passes the qvm kernel a workspace carved from a file-scope
// device array instead.
//
// The array is a fixed, modest kQvmScratchBytes (1 MiB) that every GPU which
// loads the library holds until the process exits.  Sizes whose workspace
// would not fit are rejected before any launch.  In host code the array's
// name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, on the
// first call made on it.  The address is cached for the life of the process;
// a cudaDeviceReset() reloads the module and may move the array, so calls
// after a reset of that device are not supported.
#include <mutex>

#include <cuda_runtime.h>

#include "qmv.h"
#include "qmv_launch.cuh"

namespace {

constexpr size_t kQvmScratchBytes = QMV_QVM_NOALLOC_SCRATCH_BYTES;
static_assert(kQvmScratchBytes % 256 == 0, "scratch size");

// Zero at module load; every call clears the part it uses before the kernel.
static __device__ __align__(256) unsigned char g_qvm_scratch[kQvmScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];      // device address of g_qvm_scratch, per device

// The scratch's device address on the current device (looked up once).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_qvm_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

int elem_size(int dtype) { return dtype == QMV_F32 ? 4 : 2; }

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" int qmv_qvm_affine_noalloc(const void* x, const void* w_packed, const void* scales,
                                      const void* biases, void* y, int M, int N, int K, int bits,
                                      int group_size, int dtype, void* stream) {
    if (bits != 2 && bits != 3 && bits != 4 && bits != 5 && bits != 6 && bits != 8) return QMV_EUNSUPPORTED;
    if (group_size != 32 && group_size != 64 && group_size != 128) return QMV_EUNSUPPORTED;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    if (M < 0 || M > QMV_MAX_M || N < 0 || K < 0 || N % group_size != 0) return QMV_EINVAL;
    if (M == 0 || N == 0) return QMV_OK;
    const size_t need = qmv::qvm_workspace_bytes(M, N);
    if (need > kQvmScratchBytes) return QMV_EUNSUPPORTED;          // beyond the fixed scratch
    if (!y || (K > 0 && (!x || !w_packed || !scales || !biases))) return QMV_EINVAL;
    const size_t eb = (size_t)elem_size(dtype);
    if (!is_aligned(y, eb) || (x && !is_aligned(x, eb)) || (scales && !is_aligned(scales, eb)) ||
        (biases && !is_aligned(biases, eb)) || (w_packed && !is_aligned(w_packed, 16)))
        return QMV_EALIGN;
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    // the kernel needs its partial sums and counters at zero
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QMV_ECUDA;
    }
    // the arguments are valid: the public call launches (and records a launch
    // failure for qmv_last_cuda_error)
    return qmv_qvm_affine(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, scratch, stream);
}
