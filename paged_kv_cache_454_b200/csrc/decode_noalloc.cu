// pa_decode_noalloc: paged decode for callers that cannot allocate device
// memory.
//
// Some callers have no way to hand pa_decode a workspace: a serving process
// that gives all free HBM to its KV pool at start-up (so any later cudaMalloc
// fails), or a host framework whose custom-op interface passes only inputs and
// outputs.  For them this entry point supplies the split-context scratch from
// a fixed array compiled into the library instead of from the caller.
//
// The array lives in device global memory for as long as the library is loaded
// on a device: every GPU that loads the library holds PA_NOALLOC_SCRATCH_BYTES
// until the process exits.  All calls on a device share it, and it keeps what
// the last call left in it.  Nothing in it needs to start at zero: each call's
// plan kernel rewrites the header, prefix and work list before the decode and
// merge kernels read them, and every partial result is written before it is
// read.  Two calls whose kernels overlap on the GPU (for example on two
// streams) race on the array and must not be issued.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

// Device address of the array on the current device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in, so the address is looked up
// once per device, with that device current, and cached.
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int pa_decode_noalloc(const void* q, int64_t q_stride, const void* k_pool,
                                 const void* v_pool, pa_pool_desc pool,
                                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const int32_t* context_lens, int32_t num_seqs,
                                 int32_t num_q_heads, float scale, void* out, float* lse,
                                 void* stream) {
  PA_NVTX_RANGE("pa_decode_noalloc");
  void* scratch = scratch_address();
  if (!scratch) return PA_ERR_CUDA;
  // pa_decode_ex checks every argument and returns PA_ERR_WORKSPACE, launching
  // nothing, when the batch needs more scratch than the array holds.
  return pa_decode_ex(q, q_stride, k_pool, v_pool, pool, block_tables, max_blocks_per_seq,
                      context_lens, num_seqs, num_q_heads, scale, out, lse, scratch,
                      PA_NOALLOC_SCRATCH_BYTES, 0, PA_KERNEL_AUTO, stream);
}
