// C ABI of libmsa: validation, workspace sizing and dispatch (see include/msa.h).
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace msa {

__device__ uint32_t g_device_error;

namespace {

DevCtx g_ctx[kMaxDevices];
std::mutex g_ctx_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool is_pow2_upto(int x, int maxv) {
  for (int v = 1; v <= maxv; v <<= 1)
    if (x == v) return true;
  return false;
}

// Checks shared by every op.  need_attn: head_dim/heads limits apply;
// need_index: index_dim limit applies.
msa_status check_shape(const msa_shape* s, bool need_attn, bool need_index) {
  if (!s) return MSA_ERR_NULL_PTR;
  if (s->batch < 1 || s->seq_q < 1 || s->seq_kv < 1 || s->q_offset < 0 || s->n_q_heads < 1 ||
      s->n_kv_heads < 1 || s->topk < 1)
    return MSA_ERR_INVALID_SHAPE;
  if (s->block != 128) return MSA_ERR_UNSUPPORTED;
  if (s->topk > 64) return MSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->q_offset) + s->seq_q > s->seq_kv) return MSA_ERR_INVALID_SHAPE;
  if (s->n_q_heads % s->n_kv_heads != 0) return MSA_ERR_INVALID_SHAPE;
  if (!is_pow2_upto(s->n_kv_heads, 128)) return MSA_ERR_UNSUPPORTED;   // G divides 128
  if (!is_pow2_upto(s->n_q_heads / s->n_kv_heads, 16)) return MSA_ERR_UNSUPPORTED;
  // 32-bit row indices, TMA coordinates and packed (token, slot) entries
  if (s->seq_q >= (1 << 25)) return MSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->batch) * s->seq_q * s->n_kv_heads >= (1ll << 31))
    return MSA_ERR_UNSUPPORTED;
  if (need_attn && (static_cast<int64_t>(s->batch) * s->seq_q * s->n_q_heads >= (1ll << 31) ||
                    static_cast<int64_t>(s->batch) * s->n_kv_heads * s->seq_kv >= (1ll << 31)))
    return MSA_ERR_UNSUPPORTED;
  if (need_index && static_cast<int64_t>(s->batch) * s->seq_kv >= (1ll << 31))
    return MSA_ERR_UNSUPPORTED;
  if (need_attn && s->head_dim != 64 && s->head_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (need_index && s->index_dim != 32 && s->index_dim != 64) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

msa_status check_decode(const msa_shape* s) {
  if (s->seq_q != 1 || s->q_offset != s->seq_kv - 1) return MSA_ERR_INVALID_SHAPE;
  return MSA_OK;
}

int64_t nblocks(const msa_shape& s) { return ceil_div(s.seq_kv, s.block); }

size_t pooled_bytes(const msa_shape& s) {
  return align_up(sizeof(float) * static_cast<size_t>(s.batch) * s.seq_q * s.n_kv_heads *
                      nblocks(s), 256);
}
size_t sel_bytes(const msa_shape& s) {
  return align_up(sizeof(int32_t) * static_cast<size_t>(s.batch) * s.seq_q * s.n_kv_heads *
                      s.topk, 256);
}

bool forward_is_decode(const msa_shape& s) {
  return s.seq_q == 1 && s.q_offset == s.seq_kv - 1;
}

// Pooled scores in the forward workspace: none when the prefill path fuses
// the top-k into the index scores (the selection is written directly).
size_t forward_pooled_bytes(const msa_shape& s) {
  return !forward_is_decode(s) && index_topk_fusable(s) ? 0 : pooled_bytes(s);
}

// The same for the paged chunked prefill (always the prefill path).
size_t paged_prefill_pooled_bytes(const msa_shape& s) {
  return index_topk_fusable(s, true) ? 0 : pooled_bytes(s);
}

msa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// ------------------------------------------------------------- profiling
struct ProfRecord {
  const char* name;
  cudaEvent_t a, b;
};
struct ProfEntry {
  const char* name;
  double ms;
  long long launches;
};
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<ProfRecord> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;
std::vector<ProfEntry> g_prof_table;

cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

bool prof_drain() {
  bool ok = true;
  for (const ProfRecord& r : g_prof_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      ok = false;
    ProfEntry* e = nullptr;
    for (ProfEntry& x : g_prof_table)
      if (std::strcmp(x.name, r.name) == 0) e = &x;
    if (!e) {
      g_prof_table.push_back(ProfEntry{r.name, 0.0, 0});
      e = &g_prof_table.back();
    }
    e->ms += ms;
    e->launches += 1;
    g_prof_free.push_back(r.a);
    g_prof_free.push_back(r.b);
  }
  g_prof_pending.clear();
  return ok;
}

}  // namespace

ProfScope::ProfScope(const char* name, cudaStream_t st) : st_(st) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t a = prof_event(), b = prof_event();
  if (!a || !b || cudaEventRecord(a, st) != cudaSuccess) return;
  g_prof_pending.push_back(ProfRecord{name, a, b});
  slot_ = static_cast<int>(g_prof_pending.size()) - 1;
}

ProfScope::~ProfScope() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot_ < static_cast<int>(g_prof_pending.size()))
    cudaEventRecord(g_prof_pending[slot_].b, st_);
}

const DevCtx* device_ctx() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_ctx_mu);
  DevCtx& c = g_ctx[dev];
  if (c.device < 0) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    c.err = static_cast<uint32_t*>(p);
    c.num_sms = sms;
    c.device = dev;
  }
  return &c;
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return false;
  cuuint64_t d[5];
  cuuint64_t st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d,
                        st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace msa

using namespace msa;

extern "C" {

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_SHAPE: return "MSA_ERR_INVALID_SHAPE: inconsistent shape";
    case MSA_ERR_NULL_PTR: return "MSA_ERR_NULL_PTR: a required pointer is NULL";
    case MSA_ERR_MISALIGNED: return "MSA_ERR_MISALIGNED: a device pointer is not 16-byte aligned";
    case MSA_ERR_WORKSPACE_TOO_SMALL: return "MSA_ERR_WORKSPACE_TOO_SMALL";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED: shape outside the supported limits";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA: a CUDA call or kernel launch failed";
    case MSA_ERR_DEVICE_TIMEOUT: return "MSA_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
  }
  return "MSA_ERR_UNKNOWN";
}

msa_status msa_workspace_size(const msa_shape* s, msa_op op, size_t* bytes) {
  if (!bytes) return MSA_ERR_NULL_PTR;
  *bytes = 0;
  msa_status st;
  switch (op) {
    case MSA_OP_INDEX_SCORES:
      return check_shape(s, false, true);
    case MSA_OP_BLOCK_TOPK:
      return check_shape(s, false, false);
    case MSA_OP_SPARSE_PREFILL:
      if ((st = check_shape(s, true, false)) != MSA_OK) return st;
      if (!prefill_shape_supported(*s)) return MSA_ERR_UNSUPPORTED;
      *bytes = prefill_workspace_bytes(*s);
      return MSA_OK;
    case MSA_OP_SPARSE_DECODE:
    case MSA_OP_DENSE_DECODE:
      if ((st = check_shape(s, true, false)) != MSA_OK) return st;
      if ((st = check_decode(s)) != MSA_OK) return st;
      *bytes = decode_workspace_bytes(*s, op == MSA_OP_DENSE_DECODE);
      return MSA_OK;
    case MSA_OP_FORWARD:
      if ((st = check_shape(s, true, true)) != MSA_OK) return st;
      if (!forward_is_decode(*s) && !prefill_shape_supported(*s)) return MSA_ERR_UNSUPPORTED;
      *bytes = forward_pooled_bytes(*s) + sel_bytes(*s) +
               (forward_is_decode(*s) ? decode_workspace_bytes(*s, false)
                                      : prefill_workspace_bytes(*s));
      return MSA_OK;
    case MSA_OP_DENSE_PREFILL:
      return check_shape(s, true, false);
    case MSA_OP_FORWARD_ALIGNMENT:
      if ((st = check_shape(s, true, true)) != MSA_OK) return st;
      if (!prefill_shape_supported(*s)) return MSA_ERR_UNSUPPORTED;
      *bytes = pooled_bytes(*s) + sel_bytes(*s) + prefill_workspace_bytes(*s);
      return MSA_OK;
    case MSA_OP_FORWARD_PREFILL_PAGED:
      if ((st = check_shape(s, true, true)) != MSA_OK) return st;
      if (!prefill_shape_supported(*s)) return MSA_ERR_UNSUPPORTED;
      *bytes = paged_prefill_pooled_bytes(*s) + sel_bytes(*s) + prefill_workspace_bytes(*s);
      return MSA_OK;
  }
  return MSA_ERR_UNSUPPORTED;
}

msa_status msa_index_scores(const msa_shape* s, const uint16_t* q_idx, const uint16_t* k_idx,
                            float* pooled, void* stream) {
  msa::ApiRange nvtx_("msa_index_scores");
  msa_status st = check_shape(s, false, true);
  if (st != MSA_OK) return st;
  if (!q_idx || !k_idx || !pooled) return MSA_ERR_NULL_PTR;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(pooled)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_index_scores(*s, q_idx, k_idx, pooled, true,
                                       static_cast<cudaStream_t>(stream)));
}

msa_status msa_block_topk(const msa_shape* s, const float* pooled, int32_t* sel, void* stream) {
  msa::ApiRange nvtx_("msa_block_topk");
  msa_status st = check_shape(s, false, false);
  if (st != MSA_OK) return st;
  if (!pooled || !sel) return MSA_ERR_NULL_PTR;
  if (!aligned16(pooled) || !aligned16(sel)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_block_topk(*s, pooled, sel, static_cast<cudaStream_t>(stream)));
}

static msa_status check_attn_ptrs(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const void* sel, bool need_sel, const uint16_t* o,
                                  const float* lse) {
  if (!q || !k || !v || !o || (need_sel && !sel)) return MSA_ERR_NULL_PTR;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (need_sel && !aligned16(sel)) || (lse && !aligned4(lse)))
    return MSA_ERR_MISALIGNED;
  return MSA_OK;
}

msa_status msa_sparse_attn_prefill(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                   const uint16_t* v, const int32_t* sel, uint16_t* o,
                                   float* lse, void* ws, size_t ws_bytes, void* stream) {
  msa::ApiRange nvtx_("msa_sparse_attn_prefill");
  msa_status st = check_shape(s, true, false);
  if (st != MSA_OK) return st;
  if (!prefill_shape_supported(*s)) return MSA_ERR_UNSUPPORTED;
  if ((st = check_attn_ptrs(q, k, v, sel, true, o, lse)) != MSA_OK) return st;
  const size_t need = prefill_workspace_bytes(*s);
  if (need && !ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (need && !aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_sparse_prefill(*s, q, k, v, sel, o, lse, ws,
                                         static_cast<cudaStream_t>(stream)));
}

msa_status msa_sparse_attn_decode(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const int32_t* sel, uint16_t* o,
                                  float* lse, void* ws, size_t ws_bytes, void* stream) {
  msa::ApiRange nvtx_("msa_sparse_attn_decode");
  msa_status st = check_shape(s, true, false);
  if (st != MSA_OK) return st;
  if ((st = check_decode(s)) != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, sel, true, o, lse)) != MSA_OK) return st;
  const size_t need = decode_workspace_bytes(*s, false);
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_decode(*s, q, k, v, sel, o, lse, ws, false,
                                 static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace msa {
// One decode step over caches with per-sequence lengths, contiguous
// (pages.table == nullptr) or paged: the ragged and paged entry points.
msa_status forward_decode_lens(const msa_shape* s, const int32_t* seq_lens, PageTable pages,
                               const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                               float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                               void* stream) {
  if (!s) return MSA_ERR_NULL_PTR;
  if (s->seq_q != 1) return MSA_ERR_INVALID_SHAPE;
  // seq_kv is the cache capacity; each sequence's own length comes from seq_lens
  msa_shape c = *s;
  c.q_offset = c.seq_kv - 1;
  msa_status st = check_shape(&c, true, true);
  if (st != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  if (!q_idx || !k_idx || !seq_lens) return MSA_ERR_NULL_PTR;
  if (!aligned16(q_idx) || !aligned16(k_idx) || (sel_out && !aligned16(sel_out)) ||
      !aligned4(seq_lens))
    return MSA_ERR_MISALIGNED;
  size_t need = 0;
  if ((st = msa_workspace_size(&c, MSA_OP_FORWARD, &need)) != MSA_OK) return st;
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  float* pooled = reinterpret_cast<float*>(w);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + pooled_bytes(c));
  void* rest = w + pooled_bytes(c) + sel_bytes(c);
  cudaError_t e = prepare_decode(c, rest, cs);
  if (e == cudaSuccess) e = launch_index_scores(c, q_idx, k_idx, pooled, false, cs, seq_lens, pages);
  if (e == cudaSuccess) e = launch_block_topk(c, pooled, sel, cs, seq_lens);
  if (e == cudaSuccess)
    e = launch_decode(c, q, k, v, sel, o, lse, rest, false, cs, seq_lens, pages, true);
  return from_cuda(e);
}

// Argument checks of the decode entry point without a workspace argument.
msa_status check_decode_static_args(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                    const uint16_t* v, const int32_t* sel, const uint16_t* o,
                                    const float* lse) {
  msa_status st = check_shape(s, true, false);
  if (st != MSA_OK) return st;
  if ((st = check_decode(s)) != MSA_OK) return st;
  return check_attn_ptrs(q, k, v, sel, true, o, lse);
}
}  // namespace msa

extern "C" {

msa_status msa_forward(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, const uint16_t* q_idx, const uint16_t* k_idx,
                       uint16_t* o, float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                       void* stream) {
  msa::ApiRange nvtx_("msa_forward");
  msa_status st = check_shape(s, true, true);
  if (st != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  if (!q_idx || !k_idx) return MSA_ERR_NULL_PTR;
  if (!aligned16(q_idx) || !aligned16(k_idx) || (sel_out && !aligned16(sel_out)))
    return MSA_ERR_MISALIGNED;
  size_t need = 0;
  if ((st = msa_workspace_size(s, MSA_OP_FORWARD, &need)) != MSA_OK) return st;
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const size_t pb = forward_pooled_bytes(*s);
  float* pooled = reinterpret_cast<float*>(w);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + pb);
  void* rest = w + pb + sel_bytes(*s);
  cudaError_t e;
  if (pb == 0) {
    // prefill: index scores with the top-k fused in, then the attention
    e = launch_index_topk(*s, q_idx, k_idx, sel, cs);
    if (e == cudaSuccess) e = launch_sparse_prefill(*s, q, k, v, sel, o, lse, rest, cs);
    return from_cuda(e);
  }
  const bool decode = forward_is_decode(*s);
  e = decode ? prepare_decode(*s, rest, cs) : cudaSuccess;
  if (e == cudaSuccess) e = launch_index_scores(*s, q_idx, k_idx, pooled, false, cs);
  if (e == cudaSuccess) e = launch_block_topk(*s, pooled, sel, cs);
  if (e == cudaSuccess) {
    if (decode)
      e = launch_decode(*s, q, k, v, sel, o, lse, rest, false, cs, nullptr, PageTable{}, true);
    else
      e = launch_sparse_prefill(*s, q, k, v, sel, o, lse, rest, cs);
  }
  return from_cuda(e);
}

msa_status msa_forward_alignment(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const uint16_t* q_idx,
                                 const uint16_t* k_idx, uint16_t* o, float* lse,
                                 int32_t* sel_out, float* kl, void* ws, size_t ws_bytes,
                                 void* stream) {
  msa::ApiRange nvtx_("msa_forward_alignment");
  msa_status st = check_shape(s, true, true);
  if (st != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  if (!q_idx || !k_idx || !kl) return MSA_ERR_NULL_PTR;
  if (!aligned16(q_idx) || !aligned16(k_idx) || (sel_out && !aligned16(sel_out)) || !aligned4(kl))
    return MSA_ERR_MISALIGNED;
  size_t need = 0;
  if ((st = msa_workspace_size(s, MSA_OP_FORWARD_ALIGNMENT, &need)) != MSA_OK) return st;
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  float* pooled = reinterpret_cast<float*>(w);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + pooled_bytes(*s));
  void* rest = w + pooled_bytes(*s) + sel_bytes(*s);
  cudaError_t e = launch_index_scores(*s, q_idx, k_idx, pooled, false, cs);
  if (e == cudaSuccess) e = launch_block_topk(*s, pooled, sel, cs);
  if (e == cudaSuccess) e = launch_sparse_prefill(*s, q, k, v, sel, o, lse, rest, cs, pooled, kl);
  return from_cuda(e);
}

msa_status msa_forward_decode_ragged(const msa_shape* s, const int32_t* seq_lens,
                                     const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                                     float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                                     void* stream) {
  msa::ApiRange nvtx_("msa_forward_decode_ragged");
  return forward_decode_lens(s, seq_lens, PageTable{}, q, k, v, q_idx, k_idx, o, lse, sel_out,
                             ws, ws_bytes, stream);
}

msa_status msa_forward_decode_paged(const msa_shape* s, int num_pages, const int32_t* seq_lens,
                                    const int32_t* page_table, const uint16_t* q,
                                    const uint16_t* k, const uint16_t* v, const uint16_t* q_idx,
                                    const uint16_t* k_idx, uint16_t* o, float* lse,
                                    int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  msa::ApiRange nvtx_("msa_forward_decode_paged");
  if (!s) return MSA_ERR_NULL_PTR;
  if (num_pages < 1) return MSA_ERR_INVALID_SHAPE;
  // 32-bit TMA coordinates (page*G + g) and index-key row offsets
  if (static_cast<int64_t>(num_pages) * s->n_kv_heads >= (1ll << 31) ||
      static_cast<int64_t>(num_pages) * 128 >= (1ll << 31))
    return MSA_ERR_UNSUPPORTED;
  if (!page_table) return MSA_ERR_NULL_PTR;
  if ((reinterpret_cast<uintptr_t>(page_table) & 3u) != 0) return MSA_ERR_MISALIGNED;
  PageTable pt;
  pt.table = page_table;
  pt.num_pages = num_pages;
  return forward_decode_lens(s, seq_lens, pt, q, k, v, q_idx, k_idx, o, lse, sel_out, ws,
                             ws_bytes, stream);
}

msa_status msa_forward_prefill_paged(const msa_shape* s, int num_pages,
                                     const int32_t* page_table, const uint16_t* q,
                                     const uint16_t* k, const uint16_t* v,
                                     const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                                     float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                                     void* stream) {
  msa::ApiRange nvtx_("msa_forward_prefill_paged");
  msa_status st = check_shape(s, true, true);
  if (st != MSA_OK) return st;
  if (num_pages < 1) return MSA_ERR_INVALID_SHAPE;
  // 32-bit TMA coordinates (page*G + g) and index-key rows (page*128)
  if (static_cast<int64_t>(num_pages) * s->n_kv_heads >= (1ll << 31) ||
      static_cast<int64_t>(num_pages) * 128 >= (1ll << 31))
    return MSA_ERR_UNSUPPORTED;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  if (!q_idx || !k_idx || !page_table) return MSA_ERR_NULL_PTR;
  if (!aligned16(q_idx) || !aligned16(k_idx) || (sel_out && !aligned16(sel_out)) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) != 0)
    return MSA_ERR_MISALIGNED;
  size_t need = 0;
  if ((st = msa_workspace_size(s, MSA_OP_FORWARD_PREFILL_PAGED, &need)) != MSA_OK) return st;
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  PageTable pt;
  pt.table = page_table;
  pt.num_pages = num_pages;
  char* w = static_cast<char*>(ws);
  const size_t pb = paged_prefill_pooled_bytes(*s);
  float* pooled = reinterpret_cast<float*>(w);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + pb);
  void* rest = w + pb + sel_bytes(*s);
  cudaError_t e;
  if (pb == 0) {
    e = launch_index_topk(*s, q_idx, k_idx, sel, cs, pt);
  } else {
    e = launch_index_scores(*s, q_idx, k_idx, pooled, false, cs, nullptr, pt);
    if (e == cudaSuccess) e = launch_block_topk(*s, pooled, sel, cs);
  }
  if (e == cudaSuccess)
    e = launch_sparse_prefill(*s, q, k, v, sel, o, lse, rest, cs, nullptr, nullptr, pt);
  return from_cuda(e);
}

msa_status msa_dense_attn_prefill(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, uint16_t* o, float* lse, void* ws,
                                  size_t ws_bytes, void* stream) {
  msa::ApiRange nvtx_("msa_dense_attn_prefill");
  (void)ws;
  (void)ws_bytes;
  msa_status st = check_shape(s, true, false);
  if (st != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_dense_prefill(*s, q, k, v, o, lse, static_cast<cudaStream_t>(stream)));
}

msa_status msa_dense_attn_decode(const msa_shape* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, uint16_t* o, float* lse, void* ws,
                                 size_t ws_bytes, void* stream) {
  msa::ApiRange nvtx_("msa_dense_attn_decode");
  msa_status st = check_shape(s, true, false);
  if (st != MSA_OK) return st;
  if ((st = check_decode(s)) != MSA_OK) return st;
  if ((st = check_attn_ptrs(q, k, v, nullptr, false, o, lse)) != MSA_OK) return st;
  const size_t need = decode_workspace_bytes(*s, true);
  if (!ws) return MSA_ERR_NULL_PTR;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return MSA_ERR_MISALIGNED;
  if (!device_ctx()) return MSA_ERR_CUDA;
  return from_cuda(launch_decode(*s, q, k, v, nullptr, o, lse, ws, true,
                                 static_cast<cudaStream_t>(stream)));
}

msa_status msa_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (on) {
    prof_drain();
    g_prof_table.clear();
  }
  g_prof_on.store(on != 0);
  return MSA_OK;
}

msa_status msa_profile_read(int index, const char** name, double* total_ms, long long* launches) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!prof_drain()) return MSA_ERR_CUDA;
  if (index < 0 || index >= static_cast<int>(g_prof_table.size())) return MSA_ERR_INVALID_SHAPE;
  const ProfEntry& e = g_prof_table[index];
  if (name) *name = e.name;
  if (total_ms) *total_ms = e.ms;
  if (launches) *launches = e.launches;
  return MSA_OK;
}

msa_status msa_set_wait_limit_ns(uint64_t ns) {
  if (!device_ctx()) return MSA_ERR_CUDA;
  // no kernel of the library is running when the limit changes
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = set_wait_limit_decode(ns);
  if (e == cudaSuccess) e = set_wait_limit_dense(ns);
  if (e == cudaSuccess) e = set_wait_limit_index(ns);
  if (e == cudaSuccess) e = set_wait_limit_prefill(ns);
  return from_cuda(e);
}

msa_status msa_device_status(uint32_t* flags) {
  const DevCtx* c = device_ctx();
  if (!c) return MSA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return MSA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpy(&v, c->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaMemcpy(c->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (flags) *flags = v;
  return v ? MSA_ERR_DEVICE_TIMEOUT : MSA_OK;
}

}  // extern "C"
