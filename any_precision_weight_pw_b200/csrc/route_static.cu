// route_static.cu -- pw_route_static: the router (logits, top-k, softmax and
// per-expert bucketing, the same route kernel pw_moe_forward launches) with
// its scratch in a fixed device array instead of a handle's workspace, so the
// call allocates no device memory at all.
//
// Who needs it: callers that cannot allocate device memory at the point of the
// call -- a serving loop that has handed all of HBM to weight pages and KV
// cache and must route a decode batch before any handle exists, or one that
// cannot take the device-wide synchronisation that cudaMalloc and cudaFree
// imply in the middle of an asynchronous page move.  The PagedWeight pages
// have no counterpart of this call; it is a library convenience.
//
// The scratch is one array per device for the whole process.  Its address is
// looked up with cudaGetSymbolAddress on every call made outside a stream
// capture (so a module reloaded after cudaDeviceReset is found again) and
// cached per device; a call made while its stream is being captured uses the
// cached address, so the first call on a device must come before any capture.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "pw_internal.h"

namespace {

// Carve of the scratch (every piece 256-byte aligned).
constexpr size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }
constexpr int kMaxT = PW_ROUTE_STATIC_MAX_TOKENS;
constexpr size_t kOffsetsOff = 0;
constexpr size_t kOffsetsBytes = align256(sizeof(int32_t) * (PW_MAX_EXPERTS + 2));
constexpr size_t kSlotTokOff = kOffsetsOff + kOffsetsBytes;
constexpr size_t kSlotBytes = align256(sizeof(int32_t) * kMaxT * PW_MAX_TOPK);
constexpr size_t kSlotWOff = kSlotTokOff + kSlotBytes;
constexpr size_t kTokPosOff = kSlotWOff + kSlotBytes;
constexpr size_t kTicketOff = kTokPosOff + kSlotBytes;
constexpr size_t kScratchBytes = kTicketOff + 256;
static_assert(kScratchBytes == PW_ROUTE_STATIC_SCRATCH_BYTES, "pw.h states the scratch size");

// Zero at module load; the route kernel puts its ticket back to zero at the
// end of every launch that uses it, so the next call finds it ready.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" pw_status_t pw_route_static(const uint16_t* d_x, const float* d_router_w,
                                       const float* d_router_bias, int32_t T, int32_t hidden,
                                       int32_t n_experts, int32_t top_k, int32_t renorm_topk,
                                       int32_t* d_idx, float* d_w, pw_stream_t stream) {
  if (T < 0 || T > kMaxT)
    return pw::record_error(PW_ERR_INVALID_ARG, "pw_route_static: need 0 <= T <= 256");
  if (hidden < 1 || n_experts < 1 || n_experts > PW_MAX_EXPERTS || top_k < 1 ||
      top_k > PW_MAX_TOPK || top_k > n_experts || (renorm_topk != 0 && renorm_topk != 1))
    return pw::record_error(PW_ERR_INVALID_ARG,
                            "pw_route_static: need hidden >= 1, 1 <= top_k <= min(n_experts, 8), "
                            "n_experts <= 128, renorm_topk 0 or 1");
  if (T == 0) return PW_OK;
  if (!d_x || !d_router_w || !d_idx || !d_w)
    return pw::record_error(PW_ERR_INVALID_ARG, "pw_route_static: null buffer");

  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return pw::record_error(PW_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return pw::record_error(PW_ERR_UNSUPPORTED, "pw_route_static: device ordinal >= 64");

  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap);
  if (e != cudaSuccess) return pw::record_error(PW_ERR_CUDA, cudaGetErrorString(e));
  unsigned char* base;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (cap != cudaStreamCaptureStatusNone && !g_scratch_ptr[dev])
      return pw::record_error(PW_ERR_STATE,
                              "pw_route_static: first call on a device inside a stream capture");
    if (cap == cudaStreamCaptureStatusNone) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_route_scratch);
      if (e != cudaSuccess || !p) {
        char msg[160];
        std::snprintf(msg, sizeof(msg), "pw_route_static: cudaGetSymbolAddress failed: %s",
                      cudaGetErrorString(e));
        return pw::record_error(PW_ERR_CUDA, msg);
      }
      g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
    }
    base = g_scratch_ptr[dev];
  }

  pw::RouteParams rp{};
  rp.x = d_x;
  rp.wr = d_router_w;
  rp.bias = d_router_bias;
  rp.T = T;
  rp.H = hidden;
  rp.E = n_experts;
  rp.k = top_k;
  rp.renorm = renorm_topk;
  rp.has_shared = 0;
  rp.ws.topk_idx = d_idx;
  rp.ws.topk_w = d_w;
  rp.ws.offsets = reinterpret_cast<int32_t*>(base + kOffsetsOff);
  rp.ws.slot_token = reinterpret_cast<int32_t*>(base + kSlotTokOff);
  rp.ws.slot_w = reinterpret_cast<float*>(base + kSlotWOff);
  rp.ws.token_pos = reinterpret_cast<int32_t*>(base + kTokPosOff);
  rp.ws.ticket = reinterpret_cast<uint32_t*>(base + kTicketOff);
  e = pw::launch_route(rp, n_sm, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pw::record_error(PW_ERR_CUDA, cudaGetErrorString(e));
  return PW_OK;
}

extern "C" pw_status_t pw_route_geometry(int32_t T, int32_t E, int32_t H, int32_t top_k,
                                         int64_t* out) {
  if (!out) return pw::record_error(PW_ERR_INVALID_ARG, "pw_route_geometry: null output");
  if (T < 0 || E < 1 || E > PW_MAX_EXPERTS || H < 1 || top_k < 1 || top_k > E ||
      top_k > PW_MAX_TOPK)
    return pw::record_error(PW_ERR_INVALID_ARG, "pw_route_geometry: shape out of range");
  const pw::RouteGeometry g = pw::route_geometry(T, E, H, top_k);
  const int64_t v[12] = {g.cb, g.ce, g.tb, g.tbb, g.eb, g.kc, g.n_clusters, g.tt, g.te,
                         g.sel_staged ? 1 : 0, static_cast<int64_t>(g.logits_off),
                         static_cast<int64_t>(g.smem)};
  for (int i = 0; i < 12; ++i) out[i] = v[i];
  return PW_OK;
}
