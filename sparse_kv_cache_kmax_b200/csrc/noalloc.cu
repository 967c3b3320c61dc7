// ekv_entmax_decode_static_ws: the sparse α-entmax decode for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain a scratch buffer: a plugin running
// inside a host framework that owns the whole device memory pool and hands its
// plugins no workspace, or a latency-critical serving loop that must not call
// cudaMalloc (which can synchronise the device) once it is running.  This
// entry point takes the decode's scratch from a fixed-size array compiled into
// the library instead of from the caller.  The caller still provides every
// input and output buffer.
//
// Costs and rules of the shared array (EKV_STATIC_WS_BYTES = 16 MiB):
//  * every GPU that loads libekv holds it until the process exits;
//  * every call on a device uses the same array, so calls whose work overlaps
//    on the GPU (two streams, or two host threads) race and corrupt each
//    other; serialise them;
//  * the array keeps whatever the previous call left in it.  The only scratch
//    that must start at zero is the per-unit split counter, and the first
//    decode kernel of every call sets it to zero;
//  * host code only sees a host-side stand-in for the array: the call looks
//    up its device address with the device current, the first time on a
//    device and again whenever it is made outside a stream capture (so a
//    cudaDeviceReset, which reloads the module, is followed correctly); a
//    call inside a capture uses the address found before, so make one call
//    on each device before capturing.
#include <mutex>

#include "kernels.cuh"

namespace ekv {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_decode_ws[EKV_STATIC_WS_BYTES];

std::mutex g_ws_mutex;
void* g_ws_addr[kMaxDevices] = {};

// Device address of the array on the current device.  Looked up with the
// device current on the first call, and again on every call made outside a
// stream capture (a cudaDeviceReset reloads the module, which may move the
// array); inside a capture the address found before is used, since the
// lookup is not a call to make while capturing.
cudaError_t static_ws_address(cudaStream_t stream, void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (g_ws_addr[dev] == nullptr || cap == cudaStreamCaptureStatusNone) {
    if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_decode_ws);
    if (e != cudaSuccess) return e;
    g_ws_addr[dev] = p;
  }
  *out = g_ws_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace ekv

extern "C" EKV_API ekv_status ekv_entmax_decode_static_ws(
    const ekv_cache* cache, const ekv_seqs* seqs, const void* q, int32_t num_q_heads, float scale,
    float alpha, const int32_t* sel, const int32_t* n_sel, int32_t cap, int32_t dense_v, float* out,
    float* tau, int32_t* support_count, uint32_t* support_bits, void* stream) {
  const size_t need = ekv_workspace_bytes(EKV_OP_ENTMAX_DECODE, cache, seqs, num_q_heads, cap);
  if (need == 0)  // invalid sizes: let the regular decode report which argument, before any launch
    return ekv_entmax_decode(cache, seqs, q, num_q_heads, scale, alpha, sel, n_sel, cap, dense_v,
                             out, tau, support_count, support_bits, nullptr, 0, stream);
  if (need > static_cast<size_t>(EKV_STATIC_WS_BYTES)) return EKV_ERR_WORKSPACE;
  void* ws = nullptr;
  if (ekv::static_ws_address(static_cast<cudaStream_t>(stream), &ws) != cudaSuccess) return EKV_ERR_CUDA;
  return ekv_entmax_decode(cache, seqs, q, num_q_heads, scale, alpha, sel, n_sel, cap, dense_v, out,
                           tau, support_count, support_bits, ws, EKV_STATIC_WS_BYTES, stream);
}
