// Decode attention (one query token per sequence), sparse (MSA main branch:
// yhxrc.cn article, section 第二步; lumi-systems AI news: exact block-sparse
// attention over the selected blocks) and dense causal GQA (the baseline).
//
// Split-K: one CTA per (sequence, group, split), a split being one selected
// block (sparse) or a run of consecutive causal blocks (dense).  The K and V
// rows of a block are brought into shared memory once by TMA (128-byte
// swizzle) and shared by all r = H/G query heads of the group: the heads are
// the 16 rows of an mma.sync m16n8k16 tile (zero-padded when r < 16).  Each
// warp owns 16 keys of the block and keeps its own online softmax; warps are
// merged in shared memory, splits in a last-arriving CTA chosen by an atomic
// counter (no CTA ever waits for another).  The workload is bound by HBM
// bandwidth on the K/V bytes.
#include <math.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kThreads = 256;          // 8 warps x 16 keys = one 128-key block
constexpr int kDenseBlocksPerSplit = 16;
constexpr float kLog2e = 1.4426950408889634f;

struct DecParams {
  const uint16_t* q;      // [B, 1, H, d]
  const int32_t* sel;     // [B, 1, G, k] (sparse) or nullptr (dense)
  uint16_t* o;            // [B, 1, H, d]
  float* lse;             // [B, 1, H] or nullptr
  uint32_t* counters;     // [B*G]
  float* part_lse;        // [B*G, nsplit, r]   (log2 units)
  float* part_o;          // [B*G, nsplit, r, d] normalised partial outputs
  uint32_t* err;
  int N, H, G, r, k, nsplit, bps;   // bps: blocks per split (dense)
  float scale_log2;
};

__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of element (row, col) in a [128 rows x 64 cols] bf16 tile
// written by TMA with the 128-byte swizzle (16-byte unit u of row r sits at
// unit u ^ (r & 7)); tiles of 64 columns follow each other.
__device__ __forceinline__ uint32_t sw128_off(int row, int col) {
  const int chunk = col >> 6, c = col & 63;
  const int unit = (c >> 3) ^ (row & 7);
  return static_cast<uint32_t>(chunk * (128 * 128) + row * 128 + unit * 16 + (c & 7) * 2);
}

template <int D>
__global__ void __launch_bounds__(kThreads)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  constexpr int KS = D / 16;              // k-steps of the QK^T product
  constexpr int NT = D / 8;               // n8 tiles of the PV product
  constexpr uint32_t kTile = 128u * D * 2u;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ks_ = smem;
  uint8_t* vs_ = smem + kTile;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 2 * kTile);
  float* red = reinterpret_cast<float*>(smem);   // reused after the last block
  __shared__ float wm[8][16], wl[8][16];
  __shared__ int s_last;
  __shared__ int s_abort;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qd = lane & 3;
  const int pos = p.N - 1;
  const int bt = pos >> 7;
  const int bg = b * p.G + g;

  // blocks of this split
  int blk_begin, blk_end;
  if (p.sel) {
    const int sb = p.sel[static_cast<long long>(bg) * p.k + split];
    blk_begin = sb;
    blk_end = (sb >= 0 && sb <= bt) ? sb + 1 : sb;   // empty when sb < 0
    if (sb < 0) blk_begin = blk_end = 0;
  } else {
    blk_begin = split * p.bps;
    blk_end = min(blk_begin + p.bps, bt + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // query fragments: rows = heads g*r + i (i < r), zero rows above r
  uint32_t qa[KS][4];
  {
    const uint16_t* qb = p.q + (static_cast<long long>(b) * p.H + g * p.r) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c0 = ks * 16 + 2 * qd;
      qa[ks][0] = gq < p.r ? *reinterpret_cast<const uint32_t*>(qb + gq * D + c0) : 0u;
      qa[ks][1] = gq + 8 < p.r ? *reinterpret_cast<const uint32_t*>(qb + (gq + 8) * D + c0) : 0u;
      qa[ks][2] = gq < p.r ? *reinterpret_cast<const uint32_t*>(qb + gq * D + c0 + 8) : 0u;
      qa[ks][3] =
          gq + 8 < p.r ? *reinterpret_cast<const uint32_t*>(qb + (gq + 8) * D + c0 + 8) : 0u;
    }
  }

  float m_run[2] = {-INFINITY, -INFINITY};   // rows gq, gq+8 (log2 domain)
  float l_run[2] = {0.f, 0.f};
  float o_acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o_acc[nt][0] = o_acc[nt][1] = o_acc[nt][2] = o_acc[nt][3] = 0.f;

  uint32_t phase = 0;
  bool ok = true;
  for (int blk = blk_begin; blk < blk_end && ok; ++blk, phase ^= 1u) {
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(bar, 2 * kTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(ks_ + c * 128 * 128, &tm_k, bar, c * 64, blk * 128, bg);
        tma_load_3d(vs_ + c * 128 * 128, &tm_v, bar, c * 64, blk * 128, bg);
      }
    }
    if (!mbar_wait(bar, phase, &s_abort, p.err)) ok = false;
    __syncthreads();
    if (!ok || s_abort) { ok = false; break; }
    // ---- S = Q K^T for keys kw*16 .. +15 of this block
    const uint32_t kbase = smem_u32(ks_);
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int key = warp * 16 + nt * 8 + gq;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t bb[2];
        const int col = ks * 16 + 2 * qd;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(bb[0]) : "r"(kbase + sw128_off(key, col)));
        asm volatile("ld.shared.b32 %0, [%1];"
                     : "=r"(bb[1])
                     : "r"(kbase + sw128_off(key, col + 8)));
        mma16816(s[nt], qa[ks], bb);
      }
    }
    // ---- mask, online softmax (per warp, rows gq / gq+8)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = blk * 128 + warp * 16 + nt * 8 + 2 * qd + (e & 1);
        s[nt][e] = key <= pos ? s[nt][e] * p.scale_log2 : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
      }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    }
    float corr[2], mnew[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mnew[h] = fmaxf(m_run[h], mx[h]);
      corr[h] = mnew[h] == -INFINITY ? 1.f : exp2f(m_run[h] - mnew[h]);
      m_run[h] = mnew[h];
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mh = mnew[e >> 1];
        const float pv = mh == -INFINITY ? 0.f : exp2f(s[nt][e] - mh);
        s[nt][e] = pv;
        rs[e >> 1] += pv;
      }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
      rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
      l_run[h] = l_run[h] * corr[h] + rs[h];
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      o_acc[nt][0] *= corr[0];
      o_acc[nt][1] *= corr[0];
      o_acc[nt][2] *= corr[1];
      o_acc[nt][3] *= corr[1];
    }
    // ---- O += P V  (A = P as bf16 from the S accumulators, B = V via ldmatrix.trans)
    uint32_t pa[4];
    pa[0] = pack_bf16(s[0][0], s[0][1]);
    pa[1] = pack_bf16(s[0][2], s[0][3]);
    pa[2] = pack_bf16(s[1][0], s[1][1]);
    pa[3] = pack_bf16(s[1][2], s[1][3]);
    const uint32_t vbase = smem_u32(vs_);
    const int mi = lane >> 3, ri = lane & 7;
    const int vkey = warp * 16 + (mi & 1) * 8 + ri;
#pragma unroll
    for (int nt = 0; nt < NT; nt += 2) {
      const int dcol = nt * 8 + (mi >> 1) * 8;
      uint32_t vb[4];
      ldsm_x4_trans(vbase + sw128_off(vkey, dcol), vb);
      mma16816(o_acc[nt], pa, vb);
      mma16816(o_acc[nt + 1], pa, vb + 2);
    }
    __syncthreads();   // every warp is done with this block's K/V tiles
  }

  // ---- merge the 8 warps (rows < r only)
  if (lane % 4 == 0) {
    wm[warp][gq] = m_run[0];
    wl[warp][gq] = l_run[0];
    wm[warp][gq + 8] = m_run[1];
    wl[warp][gq + 8] = l_run[1];
  }
  __syncthreads();
  float wscale[2];
  float Mrow[2], Lrow[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = gq + 8 * h;
    float M = -INFINITY;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, wm[w][row]);
    float L = 0.f;
    for (int w = 0; w < 8; ++w)
      L += wm[w][row] == -INFINITY ? 0.f : wl[w][row] * exp2f(wm[w][row] - M);
    Mrow[h] = M;
    Lrow[h] = L;
    wscale[h] = (m_run[h] == -INFINITY || L == 0.f) ? 0.f : exp2f(m_run[h] - M) / L;
  }
  // red: [8 warps][r rows][D] fp32, reusing the K/V tiles
  const int r = p.r;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int col = nt * 8 + 2 * qd;
    if (gq < r) {
      red[(warp * r + gq) * D + col] = o_acc[nt][0] * wscale[0];
      red[(warp * r + gq) * D + col + 1] = o_acc[nt][1] * wscale[0];
    }
    if (gq + 8 < r) {
      red[(warp * r + gq + 8) * D + col] = o_acc[nt][2] * wscale[1];
      red[(warp * r + gq + 8) * D + col + 1] = o_acc[nt][3] * wscale[1];
    }
  }
  __syncthreads();
  const long long part = static_cast<long long>(bg) * p.nsplit + split;
  for (int x = threadIdx.x; x < r * D; x += kThreads) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w * r * D + x];
    p.part_o[part * r * D + x] = acc;
  }
  if (threadIdx.x < 32 && lane % 4 == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = gq + 8 * h;
      if (row < r)
        p.part_lse[part * r + row] =
            (Lrow[h] > 0.f && Mrow[h] != -INFINITY) ? Mrow[h] + log2f(Lrow[h]) : -INFINITY;
    }
  }
  // ---- split combine in the last-arriving CTA of this (sequence, group)
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&p.counters[bg], 1u);
    s_last = (prev == static_cast<uint32_t>(p.nsplit - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const long long p0 = static_cast<long long>(bg) * p.nsplit;
  for (int x = threadIdx.x; x < r * D; x += kThreads) {
    const int row = x / D;
    float M = -INFINITY;
    for (int j = 0; j < p.nsplit; ++j) M = fmaxf(M, __ldcg(&p.part_lse[(p0 + j) * r + row]));
    float den = 0.f, acc = 0.f;
    for (int j = 0; j < p.nsplit; ++j) {
      const float lj = __ldcg(&p.part_lse[(p0 + j) * r + row]);
      if (lj == -INFINITY) continue;
      const float wj = exp2f(lj - M);
      den += wj;
      acc += wj * __ldcg(&p.part_o[(p0 + j) * r * D + x]);
    }
    const int h = g * r + row;
    p.o[(static_cast<long long>(b) * p.H + h) * D + (x % D)] =
        __bfloat16_as_ushort(__float2bfloat16_rn(acc / den));
    if (p.lse && (x % D) == 0)
      p.lse[static_cast<long long>(b) * p.H + h] = (M + log2f(den)) / kLog2e;
  }
  if (threadIdx.x == 0) p.counters[bg] = 0u;
}

int dense_splits(const msa_shape& s) {
  const int nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  return static_cast<int>(ceil_div(nb, kDenseBlocksPerSplit));
}

}  // namespace

size_t decode_workspace_bytes(const msa_shape& s, bool dense) {
  const int r = s.n_q_heads / s.n_kv_heads;
  const size_t bg = static_cast<size_t>(s.batch) * s.n_kv_heads;
  const size_t ns = dense ? static_cast<size_t>(dense_splits(s)) : static_cast<size_t>(s.topk);
  return align_up(bg * 4, 256) + align_up(bg * ns * r * 4, 256) +
         align_up(bg * ns * r * s.head_dim * 4, 256);
}

cudaError_t launch_decode(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* sel, uint16_t* o, float* lse,
                          void* ws, bool dense, cudaStream_t st) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  const int r = s.n_q_heads / s.n_kv_heads;
  const size_t bg = static_cast<size_t>(s.batch) * s.n_kv_heads;
  const int ns = dense ? dense_splits(s) : s.topk;
  DecParams p{};
  char* w = static_cast<char*>(ws);
  p.counters = reinterpret_cast<uint32_t*>(w);
  p.part_lse = reinterpret_cast<float*>(w + align_up(bg * 4, 256));
  p.part_o = reinterpret_cast<float*>(w + align_up(bg * 4, 256) + align_up(bg * ns * r * 4, 256));
  p.q = q;
  p.sel = dense ? nullptr : sel;
  p.o = o;
  p.lse = lse;
  p.err = ctx->err;
  p.N = s.seq_kv;
  p.H = s.n_q_heads;
  p.G = s.n_kv_heads;
  p.r = r;
  p.k = s.topk;
  p.nsplit = ns;
  p.bps = kDenseBlocksPerSplit;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(s.head_dim));

  CUtensorMap tk, tv;
  const uint64_t dims[3] = {static_cast<uint64_t>(s.head_dim), static_cast<uint64_t>(s.seq_kv),
                            static_cast<uint64_t>(bg)};
  const uint64_t strides[2] = {static_cast<uint64_t>(s.head_dim) * 2,
                               static_cast<uint64_t>(s.seq_kv) * s.head_dim * 2};
  const uint32_t box[3] = {64, 128, 1};
  if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  cudaError_t e = cudaMemsetAsync(p.counters, 0, bg * 4, st);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(ns), static_cast<unsigned>(s.n_kv_heads),
                  static_cast<unsigned>(s.batch));
  const size_t smem = 1024 + 2 * 128 * s.head_dim * 2 + 64;
  if (s.head_dim == 128) {
    e = cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
    ProfScope ps_("decode_attn", st);
    decode_attn_kernel<128><<<grid, kThreads, smem, st>>>(tk, tv, p);
  }
  } else {
    e = cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
    ProfScope ps_("decode_attn", st);
    decode_attn_kernel<64><<<grid, kThreads, smem, st>>>(tk, tv, p);
  }
  }
  return cudaGetLastError();
}

}  // namespace msa

// ------------------------------------------------ decode without allocation
// Split-K scratch of msa_sparse_attn_decode_static: one static array in
// device memory, shared by every call on a device.  Host code only ever
// passes its device address, looked up once per device.
namespace msa {
namespace {

static __device__ __align__(256) unsigned char g_decode_static_scratch[MSA_DECODE_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void* g_static_addr[64] = {};

// Device address of the scratch array on the current device (nullptr on error).
void* static_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_static_scratch) != cudaSuccess) return nullptr;
    g_static_addr[dev] = ptr;
  }
  return g_static_addr[dev];
}

}  // namespace
}  // namespace msa

extern "C" msa_status msa_sparse_attn_decode_static(const msa_shape* s, const uint16_t* q,
                                                    const uint16_t* k, const uint16_t* v,
                                                    const int32_t* sel, uint16_t* o, float* lse,
                                                    void* stream) {
  msa_status st = msa::check_decode_static_args(s, q, k, v, sel, o, lse);
  if (st != MSA_OK) return st;
  if (msa::decode_workspace_bytes(*s, false) > MSA_DECODE_STATIC_SCRATCH_BYTES)
    return MSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = msa::static_scratch_address();
  if (!scratch) return MSA_ERR_CUDA;
  const cudaError_t e = msa::launch_decode(*s, q, k, v, sel, o, lse, scratch, false,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
