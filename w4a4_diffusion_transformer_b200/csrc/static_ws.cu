// Forward pass without any allocation: the workspace is a file-scope device
// array instead of caller memory.
//
// Some callers cannot allocate device memory at the point where they run a
// layer: code that runs inside a framework's memory pool or arena without
// access to its allocator, real-time or embedded runtimes that forbid any
// allocation after start-up, and plug-ins that only receive input and output
// pointers from their host.  For them the workspace lives here, in a
// `static __device__` array of fixed size that the CUDA driver creates when the
// library's code is loaded on a device and keeps until the process exits.
//
// In host code `g_static_workspace` names a host-side stand-in, not the device
// address; the address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "svdq.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = SVDQ_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_mutex;
void* g_address[kMaxDevices] = {};

// Device address of g_static_workspace on the current device `device`.
cudaError_t static_workspace_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_address[device] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_address[device] = p;
  }
  *out = g_address[device];
  return cudaSuccess;
}

}  // namespace

extern "C" svdq_status svdq_linear_forward_static(const svdq_layer* layer, const void* X, int M, void* Y,
                                                  void* stream, unsigned flags) {
  if (!layer || !X || !Y || M < 1) return SVDQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(Y) & 15)) return SVDQ_EINVAL;
  svdq_layer_info info;
  svdq_status st = svdq_get_info(layer, &info);
  if (st != SVDQ_OK) return st;
  if (info.device < 0) return SVDQ_ESTATE;
  // the weight-only format runs without any workspace: nothing to substitute
  if (info.format == SVDQ_W4A16_INT4) return svdq_linear_forward(layer, X, M, Y, nullptr, 0, stream, flags);
  const size_t need = svdq_workspace_bytes(layer, M);
  if (need == 0) return SVDQ_EUNSUPPORTED;               // no workspace-based forward for this layer
  if (need > kStaticWorkspaceBytes) return SVDQ_EUNSUPPORTED;   // M too large for the static workspace
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return SVDQ_ECUDA;
  if (prev != info.device && cudaSetDevice(info.device) != cudaSuccess) return SVDQ_ECUDA;
  void* ws = nullptr;
  const cudaError_t e = static_workspace_address(info.device, &ws);
  if (prev != info.device) cudaSetDevice(prev);
  if (e != cudaSuccess) return SVDQ_ECUDA;
  return svdq_linear_forward(layer, X, M, Y, ws, kStaticWorkspaceBytes, stream, flags);
}
