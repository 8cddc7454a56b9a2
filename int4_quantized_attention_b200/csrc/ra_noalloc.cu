// ra_noalloc.cu -- ra_rotate_quantize_qkv_noalloc: the fused prologue with
// its scratch (error word, RoPE/rotation coefficient tables, per-channel V
// amax) held in a fixed device array of this library instead of a
// caller-provided workspace.
//
// Who needs it: callers that can hand the library their input and output
// tensors but cannot give it any extra device memory -- for example an
// engine plugin whose enqueue hook must not allocate (cudaMalloc can
// synchronise the device or fail in the middle of a run), or a program whose
// whole device memory is laid out ahead of time by a fixed arena.  This call
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library
// routine, and no host heap either.
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "ra_internal.h"

namespace {

// The scratch itself.  Every GPU that loads this library holds it until the
// process exits.  In host code `g_noalloc_scratch` only names a host-side
// stand-in, never the device memory: host code must use the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_dev[kMaxDevices] = {};                        // device address, per device
alignas(16) unsigned char g_stage[RA_NOALLOC_SCRATCH_BYTES];  // host staging of header + tables

// The array's device address on device `dev` (current), looked up on the
// device's first call and kept; a failed call drops it, so it is looked up
// again after a device reset.  Caller holds g_mutex.
cudaError_t scratch_address(int dev, char** out) {
  if (g_scratch_dev[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = ptr;
  }
  *out = static_cast<char*>(g_scratch_dev[dev]);
  return cudaSuccess;
}

ra_status cuda_err(cudaError_t e, const char* what) {
  char msg[200];
  snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
  cudaGetLastError();
  ra::set_error_detail(msg);
  return RA_ERR_CUDA;
}

}  // namespace

extern "C" ra_status ra_rotate_quantize_qkv_noalloc(const ra_problem* p, const void* q, const void* k,
                                                    const void* v, const ra_qkv4* out, ra_stream stream) {
  ra::Prob P;
  ra_status st = ra::derive_problem(p, &P);
  if (st != RA_OK) return st;
  const uintptr_t qa = reinterpret_cast<uintptr_t>(q), ka = reinterpret_cast<uintptr_t>(k),
                  va = reinterpret_cast<uintptr_t>(v);
  if (!q || !k || !v || ((qa | ka | va) & 15u)) {
    ra::set_error_detail("q, k or v NULL or not 16-byte aligned");
    return RA_ERR_INVALID_ARG;
  }
  if (out == nullptr || !out->q4 || !out->k4 || !out->v4t || !out->sq || !out->sk || !out->sv || !out->vsum ||
      ((reinterpret_cast<uintptr_t>(out->q4) | reinterpret_cast<uintptr_t>(out->k4) |
        reinterpret_cast<uintptr_t>(out->v4t) | reinterpret_cast<uintptr_t>(out->sq) |
        reinterpret_cast<uintptr_t>(out->sk) | reinterpret_cast<uintptr_t>(out->sv) |
        reinterpret_cast<uintptr_t>(out->vsum)) & 15u)) {
    ra::set_error_detail("an ra_qkv4 pointer is NULL or not 16-byte aligned");
    return RA_ERR_INVALID_ARG;
  }
  const ra::WsLayout L = ra::ws_layout(P);
  if (L.pro_bytes > RA_NOALLOC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "problem needs %zu bytes of scratch; the fixed scratch holds %u (RA_NOALLOC_SCRATCH_BYTES)",
             L.pro_bytes, (unsigned)RA_NOALLOC_SCRATCH_BYTES);
    ra::set_error_detail(msg);
    return RA_ERR_WORKSPACE;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    ra::set_error_detail("device ordinal beyond the per-device table");
    return RA_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mutex);
  char* scratch = nullptr;
  if ((e = scratch_address(dev, &scratch)) != cudaSuccess) return cuda_err(e, "cudaGetSymbolAddress");
  // Header (cleared error word + this problem's signature) and tables are
  // staged in static host memory and copied in stream order; the pageable
  // copy is staged by the runtime before cudaMemcpyAsync returns, so the
  // staging buffer may be reused by the next call.
  std::memset(g_stage, 0, L.tables);
  ra::WsHeader hdr{};
  hdr.signature = P.signature;
  std::memcpy(g_stage, &hdr, sizeof(hdr));
  ra::build_coef_tables(p, P, reinterpret_cast<float*>(g_stage + L.tables));
  e = cudaMemcpyAsync(scratch, g_stage, L.vamax, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) {
    g_scratch_dev[dev] = nullptr;   // looked up afresh next time (e.g. after a device reset)
    return cuda_err(e, "scratch upload");
  }
  // The V amax part is zeroed inside launch_prologue before it accumulates.
  e = ra::launch_prologue(P, static_cast<const __half*>(q), static_cast<const __half*>(k),
                          static_cast<const __half*>(v), out->q4, out->k4, out->v4t, out->sq, out->sk, out->sv,
                          out->vsum, scratch, s);
  if (e != cudaSuccess) {
    g_scratch_dev[dev] = nullptr;
    return cuda_err(e, "prologue launch");
  }
  return RA_OK;
}

extern "C" ra_status ra_noalloc_check_device_error(ra_stream stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    ra::set_error_detail("device ordinal beyond the per-device table");
    return RA_ERR_UNSUPPORTED;
  }
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err(e, "stream synchronize");
  char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if ((e = scratch_address(dev, &scratch)) != cudaSuccess) return cuda_err(e, "cudaGetSymbolAddress");
  }
  // the error word is the first member of the scratch's header, as in a
  // workspace; read it, and clear it when set
  ra::DeviceErr err{};
  e = cudaMemcpy(&err, scratch, sizeof(err), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(e, "error word read");
  if (err.word == 0) return RA_OK;
  e = cudaMemset(scratch, 0, sizeof(err));
  if (e != cudaSuccess) return cuda_err(e, "error word clear");
  char msg[160];
  if (err.word & ra::DEVERR_WORKSPACE) {
    snprintf(msg, sizeof(msg), "fixed scratch holds another problem's tables: overlapping calls? (site 0x%x)",
             err.site);
    ra::set_error_detail(msg);
    return RA_ERR_WORKSPACE;
  }
  snprintf(msg, sizeof(msg), "device-side check in the prologue (site 0x%x)", err.site);
  ra::set_error_detail(msg);
  return (err.word & ra::DEVERR_BOUNDS) ? RA_ERR_DEVICE_BOUNDS : RA_ERR_DEVICE_TIMEOUT;
}
