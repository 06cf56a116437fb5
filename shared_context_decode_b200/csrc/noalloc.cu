// pp_decode_attn_noalloc: decode attention for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: a plugin loaded into a host
// application that owns every device allocation and hands the plugin no
// allocator, or a serving loop that forbids device allocation after start-up
// because cudaMalloc can synchronise the device and stall unrelated streams.
// This entry point needs no workspace from them: the document pass's partial
// results go to a fixed scratch array that is part of the library itself.
//
// The array is a file-scope __device__ array, so every GPU on which the
// library's kernels are loaded holds PP_NOALLOC_SCRATCH_BYTES of it until the
// process exits.  Host code cannot use the array's name as a device address;
// the first call on each device looks the address up (cudaGetSymbolAddress,
// with that device current) and caches it.
//
// The address is kept for the life of the process; a cudaDeviceReset frees
// the array behind it, so the entry point is not for use after a reset.
//
// All calls share the one array, on every stream.  Nothing in it needs to
// start at zero (each call writes every partial it later reads), but calls
// whose kernels overlap on the GPU overwrite each other's partials: the caller
// must order them (one stream, or events).
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

static __device__ __align__(256) uint8_t g_pp_noalloc_scratch[PP_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
std::atomic<void*> g_scratch_ptr[64];

// Device address of the scratch array for the current device.
pp_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PP_ERR_CUDA;
  void* p = g_scratch_ptr[dev].load();
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_ptr[dev].load();
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_pp_noalloc_scratch) != cudaSuccess || !p) return PP_ERR_CUDA;
      g_scratch_ptr[dev].store(p);
    }
  }
  *out = p;
  return PP_OK;
}

}  // namespace

namespace {

pp_status decode_noalloc(const pp_kv_layer* layer, int32_t doc_len, const uint16_t* q,
                         const int16_t* q_sid, const int32_t* q_pos, int32_t P, float scale,
                         uint16_t* o, float* lse, const pp_options* opt, void* stream) {
  // The argument errors pp_decode_attn reports come first, with its codes.
  const pp_status v = pp::check_layer(layer);
  if (v != PP_OK) return v;
  if (P > layer->P_max) return PP_ERR_UNSUPPORTED;
  // Too much for the fixed scratch: refuse before touching anything.
  // (0 means nothing is needed, or arguments pp_decode_attn will reject.)
  if (pp_decode_workspace_bytes(P, layer->H, layer->d, doc_len, opt) > PP_NOALLOC_SCRATCH_BYTES)
    return PP_ERR_CAPACITY;
  void* scratch = nullptr;
  const pp_status s = scratch_address(&scratch);
  if (s != PP_OK) return s;
  return pp_decode_attn(layer, doc_len, q, q_sid, q_pos, P, scale, o, lse, scratch,
                        PP_NOALLOC_SCRATCH_BYTES, opt, stream);
}

}  // namespace

extern "C" __attribute__((visibility("default"))) pp_status pp_decode_attn_noalloc(
    const pp_kv_layer* layer, int32_t doc_len, const uint16_t* q, const int16_t* q_sid,
    const int32_t* q_pos, int32_t P, float scale, uint16_t* o, float* lse, const pp_options* opt,
    void* stream) {
  nvtxRangePushA("pp_decode_attn_noalloc");
  const pp_status st = decode_noalloc(layer, doc_len, q, q_sid, q_pos, P, scale, o, lse, opt, stream);
  nvtxRangePop();
  return st;
}
