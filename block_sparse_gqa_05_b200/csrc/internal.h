// Host-side declarations shared by the translation units of libmsa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

#include "msa.h"

namespace msa {

// Most devices a process may use the library on (per-device tables are this long).
constexpr int kMaxDevices = 64;

// Per-device context: the device error word (a __device__ symbol) and SM count.
// Looked up once per device and kept for the life of the process: after a
// cudaDeviceReset the cached device addresses are stale, so a process that
// resets a device must not call the library on it again.
struct DevCtx {
  uint32_t* err = nullptr;
  int num_sms = 0;
  int device = -1;
};

// Returns nullptr if the CUDA runtime cannot be queried.
const DevCtx* device_ctx();

// TMA descriptor encoding through the driver entry point (no -lcuda link).
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);

// Brackets one kernel launch with CUDA events when profiling is enabled.
class ProfScope {
 public:
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int slot_ = -1;
  cudaStream_t st_ = nullptr;
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// An NVTX range around each compute call of the C ABI (a timeline tool shows
// the call with its kernels under it; without a tool attached it costs a
// pointer test).
struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};

// Launches a kernel that may start before the previous kernel on the stream
// has finished (programmatic dependent launch); the kernel itself waits
// (griddepcontrol.wait) before reading that kernel's results.  Captured into
// CUDA graphs as a programmatic edge.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.  Shapes are already validated.
// lens (device, [B], may be null): per-sequence cache lengths of ragged decode;
// the query of sequence b then sits at position lens[b] - 1.
// Paged caches (decode): one 128-row block per page, table [B, nb] of page
// ids; k_idx then holds [num_pages, 128, d_i] rows and k, v [num_pages, G,
// 128, d].  table == nullptr: contiguous caches.
struct PageTable {
  const int32_t* table = nullptr;
  int num_pages = 0;
};
cudaError_t launch_index_scores(const msa_shape& s, const uint16_t* q_idx,
                                const uint16_t* k_idx, float* pooled, bool fill_upper,
                                cudaStream_t st, const int32_t* lens = nullptr,
                                PageTable pages = PageTable{});
// Index scores with the block top-k fused in (prefill shapes on the tensor-core
// path, k <= 32): writes the selection directly, no pooled scores.
bool index_topk_fusable(const msa_shape& s, bool paged = false);
cudaError_t launch_index_topk(const msa_shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                              int32_t* sel, cudaStream_t st, PageTable pages = PageTable{});
cudaError_t launch_block_topk(const msa_shape& s, const float* pooled, int32_t* sel,
                              cudaStream_t st, const int32_t* lens = nullptr);
size_t prefill_workspace_bytes(const msa_shape& s);
// Shared-memory limits of the prefill path's per-CTA tables: the inversion's
// [2 nb] histogram and the combine's [k][H] (max, sum) pairs plus its [G][k]
// entry map (and, with the alignment output, [H] head sums and [G][k] pooled
// scores).  False when a shape needs more than one CTA can hold.
bool prefill_shape_supported(const msa_shape& s);
// Paged caches (chunked prefill): k, v [num_pages, G, 128, d] with the table
// [B, nb]; the V rows of a sequence's last page past N are zeroed before use.
cudaError_t launch_sparse_prefill(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const int32_t* sel, uint16_t* o,
                                  float* lse, void* ws, cudaStream_t st,
                                  const float* pooled = nullptr, float* kl = nullptr,
                                  PageTable pages = PageTable{});
size_t decode_workspace_bytes(const msa_shape& s, bool dense);
cudaError_t launch_decode(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* sel, uint16_t* o, float* lse,
                          void* ws, bool dense, cudaStream_t st,
                          const int32_t* lens = nullptr, PageTable pages = PageTable{},
                          bool counters_zeroed = false);
// Zeroes the decode workspace's per-(sequence, group) counters ahead of the
// kernels that precede the attention, so that the attention kernel follows
// the top-k directly on the stream (and may start while it finishes); then
// launch_decode(..., counters_zeroed = true).
cudaError_t prepare_decode(const msa_shape& s, void* ws, cudaStream_t st);
msa_status check_decode_static_args(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                    const uint16_t* v, const int32_t* sel, const uint16_t* o,
                                    const float* lse);
// The bounded waits' limit of each kernel translation unit, on the current
// device (msa_set_wait_limit_ns).
cudaError_t set_wait_limit_decode(uint64_t ns);
cudaError_t set_wait_limit_dense(uint64_t ns);
cudaError_t set_wait_limit_index(uint64_t ns);
cudaError_t set_wait_limit_prefill(uint64_t ns);
cudaError_t launch_dense_prefill(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, uint16_t* o, float* lse, cudaStream_t st);

}  // namespace msa
