// C ABI entry points of libpa that are not kernels themselves: argument
// checks, workspace carving, kernel choice, the device error word.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "../../include/pa_kv_manager.h"

namespace pa {

// The sticky per-device error word the kernels OR their PA_DEV_ERR_* bits into.
__device__ unsigned int g_device_error_word;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}
}  // namespace

unsigned int* device_error_word() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_err_ptr[dev];
}

int num_sms() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

int KernelLaunchCache::blocks_per_sm(const void* func, int threads, int smem_bytes) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!per_sm[dev]) {
    if (smem_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
            cudaSuccess)
      return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem_bytes) !=
            cudaSuccess ||
        n < 1)
      return 0;
    per_sm[dev] = n;
  }
  return per_sm[dev];
}

int check_pool(const pa_pool_desc& pool) {
  if (pool.num_blocks <= 0 || pool.num_kv_heads <= 0) return PA_ERR_SHAPE;
  if (pool.block_size != 16) return PA_ERR_UNSUPPORTED;
  if (pool.head_dim != 64 && pool.head_dim != 128) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Runs of at least two sequences: at most num_seqs / 2 of them.
static size_t max_runs(int S) { return size_t(S) / 2 + 1; }

size_t decode_workspace_bytes(int S, int Hq, int Hkv, int D, int max_parts) {
  const size_t slots = size_t(S) * (size_t(max_parts) + 1);
  size_t b = align256(8 * sizeof(int));
  b += align256(sizeof(int) * (size_t(S) + 1));
  b += align256(sizeof(int) * size_t(S) * size_t(Hkv));
  b += align256(sizeof(int2) * slots * size_t(Hkv));
  b += 2 * align256(sizeof(int) * size_t(S));
  b += align256(sizeof(int) * max_runs(S) * kRunInts);
  b += align256(sizeof(int2) * max_runs(S) * size_t(Hkv) * size_t(max_parts));
  b += align256(sizeof(float) * slots * size_t(Hq) * size_t(D));
  b += align256(sizeof(float) * slots * size_t(Hq));
  return b;
}

DecodeWorkspace carve_decode_workspace(void* ws, int S, int Hq, int Hkv, int D, int max_parts) {
  const size_t slots = size_t(S) * (size_t(max_parts) + 1);
  char* p = static_cast<char*>(ws);
  DecodeWorkspace w;
  w.header = reinterpret_cast<int*>(p);
  p += align256(8 * sizeof(int));
  w.part_base = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t(S) + 1));
  w.merge_cnt = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * size_t(S) * size_t(Hkv));
  w.items = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * slots * size_t(Hkv));
  w.seq_span = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * size_t(S));
  w.seq_pp = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * size_t(S));
  w.runs = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * max_runs(S) * kRunInts);
  w.pitems = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * max_runs(S) * size_t(Hkv) * size_t(max_parts));
  w.part_o = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * slots * size_t(Hq) * size_t(D));
  w.part_lse = reinterpret_cast<float*>(p);
  return w;
}

}  // namespace pa

using namespace pa;

namespace {

// Shortest default partition of the tensor-core kernel: kTcPartition tokens of
// one KV head, i.e. the same bytes per item when an item packs several heads.
int tc_min_partition(int item_heads) {
  const int p = kTcPartition / item_heads;
  return p < 128 ? 128 : p;
}

int partition_or_default(int partition_tokens, int kernel, int item_heads) {
  if (partition_tokens > 0) return partition_tokens;
  return kernel == PA_KERNEL_TCGEN05 ? tc_min_partition(item_heads) : kSimtPartition;
}

int max_parts_for(int max_blocks, int block_size, int partition_tokens) {
  const long long max_ctx = static_cast<long long>(max_blocks) * block_size;
  long long p = (max_ctx + partition_tokens - 1) / partition_tokens;
  return static_cast<int>(p < 1 ? 1 : p);
}

int choose_kernel(int kernel, int head_dim, int group) {
  if (kernel == PA_KERNEL_AUTO)
    return decode_tcgen05_supported(head_dim, group) ? PA_KERNEL_TCGEN05 : PA_KERNEL_SIMT;
  return kernel;
}

}  // namespace

extern "C" {

size_t pa_decode_workspace_size_ex(int32_t num_seqs, int32_t num_q_heads, pa_pool_desc pool,
                                   int32_t max_blocks_per_seq, int32_t partition_tokens) {
  if (num_seqs < 0 || num_q_heads <= 0 || pool.num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      pool.block_size <= 0 || pool.head_dim <= 0)
    return 0;
  // Size for the smaller of the two defaults when the caller leaves the choice
  // to the library, so either kernel fits.
  int part = partition_tokens;
  if (part <= 0) {
    part = kSimtPartition;
    const int group = num_q_heads / pool.num_kv_heads;
    if (group >= 1 && num_q_heads % pool.num_kv_heads == 0 &&
        decode_tcgen05_supported(pool.head_dim, group)) {
      const int tc = tc_min_partition(decode_tcgen05_heads_per_item(group, pool.num_kv_heads));
      if (tc < part) part = tc;
    }
  }
  const int mp = max_parts_for(max_blocks_per_seq, pool.block_size, part);
  return decode_workspace_bytes(num_seqs, num_q_heads, pool.num_kv_heads, pool.head_dim, mp);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, pa_pool_desc pool,
                                int32_t max_blocks_per_seq) {
  return pa_decode_workspace_size_ex(num_seqs, num_q_heads, pool, max_blocks_per_seq, 0);
}

int pa_decode_ex(const void* q, int64_t q_stride, const void* k_pool, const void* v_pool,
                 pa_pool_desc pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                 const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                 int32_t partition_tokens, int32_t kernel, void* stream) {
  PA_NVTX_RANGE("pa_decode_ex");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0) return PA_ERR_ARG;
  if (num_q_heads % pool.num_kv_heads) return PA_ERR_SHAPE;
  const int group = num_q_heads / pool.num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if (kernel < PA_KERNEL_AUTO || kernel > PA_KERNEL_TCGEN05) return PA_ERR_ARG;
  if (partition_tokens < 0 || (partition_tokens > 0 && partition_tokens % 128)) return PA_ERR_ARG;
  if (partition_tokens > 0 && partition_tokens < 128) return PA_ERR_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out) return PA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PA_ERR_ARG;
  if (q_stride < static_cast<int64_t>(num_q_heads) * pool.head_dim || q_stride % 8)
    return PA_ERR_ARG;
  const int kind = choose_kernel(kernel, pool.head_dim, group);
  if (kind == PA_KERNEL_TCGEN05 && !decode_tcgen05_supported(pool.head_dim, group))
    return PA_ERR_UNSUPPORTED;
  const int item_heads =
      kind == PA_KERNEL_TCGEN05 ? decode_tcgen05_heads_per_item(group, pool.num_kv_heads) : 1;
  int part = partition_or_default(partition_tokens, kind, item_heads);
  {
    // a partition longer than any context the table can describe is one partition
    const long long max_ctx = static_cast<long long>(max_blocks_per_seq) * pool.block_size;
    const long long cap = ((max_ctx + 127) / 128) * 128;
    if (part > cap) part = static_cast<int>(cap < 128 ? 128 : cap);
  }
  const int max_parts = max_parts_for(max_blocks_per_seq, pool.block_size, part);
  // work items carry (KV-head group << 16 | partition) in one int32
  if (max_parts > 0xffff || pool.num_kv_heads > 0x7fff) return PA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(num_seqs, num_q_heads, pool.num_kv_heads,
                                             pool.head_dim, max_parts);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;

  DecodeArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.q_stride = q_stride;
  a.k_pool = static_cast<const uint16_t*>(k_pool);
  a.v_pool = static_cast<const uint16_t*>(v_pool);
  a.pool = pool;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.scale = scale;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  if (partition_tokens > 0) {
    a.min_part = a.max_part = part;  // the caller fixed the length
  } else {
    a.min_part = part;
    if (kind == PA_KERNEL_TCGEN05) {
      const int mx = kTcMaxPartition / item_heads;
      a.max_part = mx > part ? mx : part;
    } else {
      a.max_part = part;
    }
  }
  a.target_items = kTcItemsPerSm * num_sms();
  a.max_parts = max_parts;
  a.ws = carve_decode_workspace(workspace, num_seqs, num_q_heads, pool.num_kv_heads,
                                pool.head_dim, max_parts);
  a.err = device_error_word();
  a.stream = as_stream(stream);
  if (!a.err) return PA_ERR_CUDA;
  a.item_heads = item_heads;
  // shared prefixes read once for all their sharers (tensor-core kernel, and
  // batches the plan can sort): items of 8 q columns, so groups up to 4 (two
  // sharers at least), run in the same launch as the sequences' own items
  a.casc_cols = 0;
  if (kind == PA_KERNEL_TCGEN05 && num_seqs >= 2 && num_seqs <= kCascMaxSeqs && group <= 4)
    a.casc_cols = 8;

  st = launch_decode_plan(a);
  if (st != PA_OK) return st;
  if (kind == PA_KERNEL_TCGEN05) return launch_decode_tcgen05(a);
  st = launch_decode_simt(a);
  if (st != PA_OK) return st;
  return launch_decode_merge(a);
}

int pa_decode(const void* q, int64_t q_stride, const void* k_pool, const void* v_pool,
              pa_pool_desc pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
              const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
              void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  PA_NVTX_RANGE("pa_decode");
  return pa_decode_ex(q, q_stride, k_pool, v_pool, pool, block_tables, max_blocks_per_seq,
                      context_lens, num_seqs, num_q_heads, scale, out, lse, workspace,
                      workspace_bytes, 0, PA_KERNEL_AUTO, stream);
}

int pa_chunked_prefill(const void* q, int64_t q_stride, const int32_t* cu_q_lens,
                       int32_t total_q, int32_t max_q_len, const void* k_pool,
                       const void* v_pool, pa_pool_desc pool, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, const int32_t* context_lens,
                       int32_t num_seqs, int32_t num_q_heads, float scale, void* out, float* lse,
                       void* stream) {
  PA_NVTX_RANGE("pa_chunked_prefill");
  return pa_chunked_prefill_ex(q, q_stride, cu_q_lens, total_q, max_q_len, k_pool, v_pool, pool,
                               block_tables, max_blocks_per_seq, context_lens, num_seqs,
                               num_q_heads, scale, out, lse, 0u, stream);
}

int pa_chunked_prefill_ex(const void* q, int64_t q_stride, const int32_t* cu_q_lens,
                          int32_t total_q, int32_t max_q_len, const void* k_pool,
                          const void* v_pool, pa_pool_desc pool, const int32_t* block_tables,
                          int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_q_heads, float scale, void* out,
                          float* lse, uint32_t flags, void* stream) {
  PA_NVTX_RANGE("pa_chunked_prefill_ex");
  if (flags & ~static_cast<uint32_t>(PA_PREFILL_EXACT_WEIGHTS)) return PA_ERR_ARG;
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || num_q_heads <= 0 ||
      max_blocks_per_seq <= 0)
    return PA_ERR_ARG;
  if (num_q_heads % pool.num_kv_heads) return PA_ERR_SHAPE;
  if (num_q_heads / pool.num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || total_q == 0) return PA_OK;
  if (!q || !cu_q_lens || !k_pool || !v_pool || !block_tables || !context_lens || !out)
    return PA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PA_ERR_ARG;
  if (q_stride < static_cast<int64_t>(num_q_heads) * pool.head_dim || q_stride % 8)
    return PA_ERR_ARG;
  PrefillArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.q_stride = q_stride;
  a.cu_q = cu_q_lens;
  a.total_q = total_q;
  a.max_q_len = max_q_len;
  a.k_pool = static_cast<const uint16_t*>(k_pool);
  a.v_pool = static_cast<const uint16_t*>(v_pool);
  a.pool = pool;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.scale = scale;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.exact_weights = (flags & PA_PREFILL_EXACT_WEIGHTS) != 0;
  a.err = device_error_word();
  a.stream = as_stream(stream);
  if (!a.err) return PA_ERR_CUDA;
  if (prefill_tcgen05_supported(a)) return launch_prefill_tcgen05(a);
  return launch_prefill_simt(a);
}

int pa_get_device_error(uint32_t* flags_host, void* stream) {
  PA_NVTX_RANGE("pa_get_device_error");
  if (!flags_host) return PA_ERR_ARG;
  unsigned int* w = device_error_word();
  if (!w) return PA_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  unsigned int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemset(w, 0, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  *flags_host = v;
  return PA_OK;
}

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_ARG: return "PA_ERR_ARG: bad argument (null, negative, misaligned)";
    case PA_ERR_SHAPE: return "PA_ERR_SHAPE: inconsistent sizes";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: size not compiled";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing or too small";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime or launch failure";
    case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS: too few free blocks in the pool";
    default: return "unknown status";
  }
}

int pa_abi_version(void) { return PA_ABI_VERSION; }

}  // extern "C"
