// Attention forward for callers that cannot allocate device memory.
//
// hstu_attention_fwd needs a caller-provided workspace (the tensor-core
// kernel's longest-first work list).  Some callers have no allocator to get
// it from: processes that run under a fixed device-memory budget planned at
// start-up and may not allocate on their request path, and plain C hosts that
// own only their input and output buffers.  This entry point takes the same
// inputs and outputs but keeps its scratch in the static array below, which
// every GPU that loads the library holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

// Maximum scratch: 2 MiB.  The work list needs 6,400 bytes of counters plus
// 8 bytes per (128-query tile, head) item, (T / 128 + B + 1) * H items, so it
// holds up to 261,344 items.
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on the current device.  Looked up once
// per device, with that device current; the host-side symbol itself is only
// a stand-in and must never be passed to a kernel.  The cached address stays
// valid for the life of the device's primary context: a process that resets
// the device (cudaDeviceReset) must not call this entry point afterwards.
void* noalloc_scratch(int* err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *err = 1;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *err = 1;
      return nullptr;
    }
    g_noalloc_ptr[dev] = p;
  }
  *err = 0;
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" hstu_status hstu_attention_fwd_noalloc(const hstu_config* cfg, const float* rab_pos,
                                                  const float* rab_time, const void* g,
                                                  const int64_t* seq_offsets, int32_t B, int64_t T,
                                                  const int64_t* timestamps,
                                                  const int32_t* num_targets, void* o_out,
                                                  cudaStream_t stream) {
  // The checks of the allocating entry point, run with a zero-sized
  // workspace: they report argument errors without touching the device.
  // (a zero-sized workspace always fails its size check, so a well-formed
  // call comes back with HSTU_ERR_WORKSPACE here).
  const hstu_status st = hstu_attention_fwd(cfg, rab_pos, rab_time, g, seq_offsets, B, T,
                                            timestamps, num_targets, o_out, nullptr, 0, stream);
  if (st != HSTU_ERR_WORKSPACE) return st;
  if (B == 0 || T == 0) return HSTU_OK;  // nothing to compute; the scratch is not touched
  // The work list must fit; bf16 heads of 32 also use the scratch left after
  // it for their zero-padded copy when that fits too (else the CUDA-core kernel).
  const size_t need = hstu::attention_fwd_ws(B, T, cfg->num_heads);
  if (need > kNoAllocScratchBytes) return HSTU_ERR_WORKSPACE;  // beyond the static scratch
  int err = 0;
  void* ws = noalloc_scratch(&err);
  if (err) return HSTU_ERR_CUDA;
  // The work list is rebuilt (and its counters cleared) by every call.
  return hstu_attention_fwd(cfg, rab_pos, rab_time, g, seq_offsets, B, T, timestamps, num_targets,
                            o_out, ws, kNoAllocScratchBytes, stream);
}
