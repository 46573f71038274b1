// Host-side declarations shared by the translation units of libpa.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pa.h"

#ifndef PA_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace pa {

// Device address of the sticky error word of the current device (looked up
// once per device with cudaGetSymbolAddress).  NULL if the lookup failed.
unsigned int* device_error_word();

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// An NVTX range around one C-ABI call (named after the entry point), so a
// profiler timeline shows which library call each kernel belongs to.  NVTX is
// header-only: without a profiler attached a push/pop costs a few nanoseconds
// and loads nothing.  -DPA_NO_NVTX compiles the ranges out.
#ifndef PA_NO_NVTX
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define PA_NVTX_RANGE(name) ::pa::NvtxRange pa_nvtx_range_(name)
#else
#define PA_NVTX_RANGE(name) ((void)0)
#endif

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-kernel, per-device launch facts: sets the dynamic shared-memory limit
// once per device and caches the occupancy (resident CTAs per SM).
struct KernelLaunchCache {
  int per_sm[64] = {0};
  int blocks_per_sm(const void* func, int threads, int smem_bytes);
};

// Host checks of a pool descriptor shared by every entry point.
int check_pool(const pa_pool_desc& pool);

// Launch status -> PA status.
inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Decode: the work plan shared by the decode kernels and the merge.
// ---------------------------------------------------------------------------
// The workspace holds, in order:
//   header       int32[8]: total items, total partitions, dynamic item counter,
//                partition length chosen by the plan, shared-prefix items,
//                their dynamic counter, log2 of the KV heads per shared-prefix
//                item, the shared prefixes' partition length
//   part_base    int32[num_seqs + 1]: exclusive prefix of partitions per sequence
//   merge_cnt    int32[num_seqs * Hkv]: partitions finished per (sequence, KV head)
//   work list    int2[num_seqs * max_parts * Hkv]: (seq, head group << 16 | partition)
//                in the plan's order; a head group is item_heads KV heads; the
//                partition counts from the end of the sequence's shared prefix
//   seq_span     int32[num_seqs]: tokens of the sequence's shared prefix (0: none)
//   seq_pp       int32[num_seqs]: partitions of that prefix
//   runs         int32[num_seqs / 2 * kRunInts]: per run of sequences sharing a
//                prefix: its length in tokens, its member count, the members
//   prefix list  int2[num_seqs / 2 * Hkv * max_parts]: (run, head group << 16 |
//                partition) of the shared-prefix items
//   partial out  float[num_seqs * (max_parts + 1) * Hq * D]
//   partial lse  float[num_seqs * (max_parts + 1) * Hq]   (base-2 log-sum-exp)
// max_parts is the partition count of the longest possible context at the
// shortest partition length the call may use; a sequence with a shared prefix
// may have one partition more (the prefix and the rest are split separately).
constexpr int kRunInts = 18;  // span, members, up to 16 member sequences
struct DecodeWorkspace {
  int* header;
  int* part_base;
  int* merge_cnt;
  int2* items;
  int* seq_span;
  int* seq_pp;
  int* runs;
  int2* pitems;
  float* part_o;
  float* part_lse;
};

size_t decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                              int max_parts);
DecodeWorkspace carve_decode_workspace(void* ws, int num_seqs, int num_q_heads,
                                       int num_kv_heads, int head_dim, int max_parts);

struct DecodeArgs {
  const uint16_t* q;
  int64_t q_stride;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  pa_pool_desc pool;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int num_seqs;
  int num_q_heads;
  float scale;
  uint16_t* out;
  float* lse;
  int min_part;      // partition length bounds for the plan (tokens, multiples of 128)
  int max_part;
  int target_items;  // the plan lengthens partitions while at least this many items remain
  int max_parts;     // workspace bound (partitions of the longest context at min_part)
  int item_heads = 1;  // KV heads per work item (the tensor-core kernel packs small groups)
  // Shared-prefix cascade (tensor-core kernel): sequences that share their
  // first blocks read the shared span once, in items whose casc_cols q columns
  // are the sharers' q heads (the plan picks the sharers and KV heads per
  // item).  0: no cascade.
  int casc_cols = 0;
  DecodeWorkspace ws;
  unsigned int* err;
  cudaStream_t stream;
};

// Kernel launchers (return PA_OK / PA_ERR_*).
int launch_decode_plan(const DecodeArgs& a);
int launch_decode_simt(const DecodeArgs& a);
int launch_decode_tcgen05(const DecodeArgs& a);  // merges split partitions itself
int launch_decode_merge(const DecodeArgs& a);

// Partition lengths (tokens) of the two decode kernels: the CUDA-core kernel
// uses a fixed length; the tensor-core kernel starts from kTcPartition (of one
// KV head) and lengthens partitions up to kTcMaxPartition while each SM keeps
// at least kTcItemsPerSm items (longest-first order keeps the tail short, and
// every item has a fixed cost: a sweep of fixed lengths on B200 found the
// longest such length fastest on the 7B-, 70B- and mixed-shaped batches).
constexpr int kSimtPartition = 512;
constexpr int kTcPartition = 1024;
constexpr int kTcMaxPartition = 8192;
constexpr int kTcItemsPerSm = 2;
// The plan finds shared prefixes in batches of up to this many sequences.
constexpr int kCascMaxSeqs = 1024;

struct PrefillArgs {
  const uint16_t* q;
  int64_t q_stride;
  const int32_t* cu_q;
  int total_q;
  int max_q_len;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  pa_pool_desc pool;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int num_seqs;
  int num_q_heads;
  float scale;
  uint16_t* out;
  float* lse;
  bool exact_weights = false;  // PA_PREFILL_EXACT_WEIGHTS
  unsigned int* err;
  cudaStream_t stream;
};

int launch_prefill_simt(const PrefillArgs& a);
int launch_prefill_tcgen05(const PrefillArgs& a);
bool prefill_tcgen05_supported(const PrefillArgs& a);
bool decode_tcgen05_supported(int head_dim, int group);
// KV heads the tensor-core decode kernel puts in one work item (a power of two
// dividing hkv).
int decode_tcgen05_heads_per_item(int group, int hkv);

}  // namespace pa
