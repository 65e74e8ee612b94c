// Main branch, prefill: exact softmax attention over the selected blocks
// (yhxrc.cn article, section 第二步: Q/K/V keep the GQA shapes, only the blocks
// listed in I_g are read, every head of group g shares I_g; lumi-systems AI
// news: exact block-sparse attention with a "KV-outer" loop so the tensor
// cores work at block granularity).
//
// Schedule (KV-outer):
//  1. invert sel: for every (sequence, group, block) column, the list of
//     (token, slot) pairs that selected it (counting sort in three passes);
//  2. cut every column into tiles of 128/r tokens = 128 (token, head) rows;
//  3. persistent tcgen05 kernel: each selected K/V block is TMA-loaded once per
//     CTA that works on it and reused by every tile of its column; for a tile,
//     S = Q K^T (TMEM), softmax over the block (causal mask on the local
//     block), P (bf16, smem) , O_part = P V (TMEM) -> normalised bf16 partial
//     and its log-sum-exp per (token, head, slot);
//  4. combine the k partials of every (token, head) by their log-sum-exp.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAttnThreads = 192;   // warp 0: TMA, warp 1: MMA, warps 2..5: softmax/epilogue
constexpr int kHistTokens = 1024;   // tokens per CTA of the inversion passes

struct PrefillWs {
  uint32_t* col_count;   // [ncol]
  uint32_t* col_fill;    // [ncol]
  uint32_t* col_off;     // [ncol + 1]
  uint32_t* tile_off;    // [ncol + 1]
  uint32_t* entries;     // [B*T*G*k]   (t << 6) | slot
  int4* tiles;           // [max_tiles] (column, entry start, count, 0)
  uint16_t* part_o;      // [B, T, k, H, d] bf16, normalised partial outputs
  float* part_lse;       // [B, T, k, H]    log-sum-exp of each partial, log2 units
  long long ncol, max_tiles;
};

PrefillWs carve(const msa_shape& s, void* base) {
  PrefillWs w{};
  const long long nb = ceil_div(s.seq_kv, 128);
  const int r = s.n_q_heads / s.n_kv_heads;
  const int tpt = 128 / r;
  w.ncol = static_cast<long long>(s.batch) * s.n_kv_heads * nb;
  const long long nent = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads * s.topk;
  w.max_tiles = ceil_div(nent, tpt) + w.ncol;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = p ? p + off : nullptr;
    off += align_up(bytes, 256);
    return q;
  };
  w.col_count = reinterpret_cast<uint32_t*>(take(4 * w.ncol));
  w.col_fill = reinterpret_cast<uint32_t*>(take(4 * w.ncol));
  w.col_off = reinterpret_cast<uint32_t*>(take(4 * (w.ncol + 1)));
  w.tile_off = reinterpret_cast<uint32_t*>(take(4 * (w.ncol + 1)));
  w.entries = reinterpret_cast<uint32_t*>(take(4 * nent));
  w.tiles = reinterpret_cast<int4*>(take(16 * w.max_tiles));
  w.part_o = reinterpret_cast<uint16_t*>(take(2ull * s.batch * s.seq_q * s.n_q_heads *
                                              s.topk * s.head_dim));
  w.part_lse = reinterpret_cast<float*>(take(4ull * s.batch * s.seq_q * s.n_q_heads * s.topk));
  return w;
}

size_t carve_bytes(const msa_shape& s) {
  const long long nb = ceil_div(s.seq_kv, 128);
  const int r = s.n_q_heads / s.n_kv_heads;
  const int tpt = 128 / r;
  const long long ncol = static_cast<long long>(s.batch) * s.n_kv_heads * nb;
  const long long nent = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads * s.topk;
  const long long max_tiles = ceil_div(nent, tpt) + ncol;
  size_t b = 0;
  b += align_up(4 * ncol, 256) * 2;
  b += align_up(4 * (ncol + 1), 256) * 2;
  b += align_up(4 * nent, 256);
  b += align_up(16 * max_tiles, 256);
  b += align_up(2ull * s.batch * s.seq_q * s.n_q_heads * s.topk * s.head_dim, 256);
  b += align_up(4ull * s.batch * s.seq_q * s.n_q_heads * s.topk, 256);
  return b;
}

// ------------------------------------------------------- 1. invert selection
// grid: (ceil(T / kHistTokens), B*G).  Pass 0 counts (sequence, group, block)
// hits; pass 1 reserves a range per column and scatters (token, slot) entries.
__global__ void __launch_bounds__(256) sel_invert_kernel(const int32_t* __restrict__ sel,
                                                         PrefillWs w, int T, int G, int k,
                                                         int nb, int pass) {
  extern __shared__ uint32_t hist[];   // [nb] counts, then [nb] cursors/bases
  uint32_t* base = hist + nb;
  const int bg = blockIdx.y;
  const int b = bg / G, g = bg % G;
  const int t0 = blockIdx.x * kHistTokens;
  const int t1 = min(T, t0 + kHistTokens);
  for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  for (int x = threadIdx.x; x < (t1 - t0) * k; x += blockDim.x) {
    const int t = t0 + x / k, slot = x % k;
    const int c = sel[((static_cast<long long>(b) * T + t) * G + g) * k + slot];
    if (c >= 0) atomicAdd(&hist[c], 1u);
  }
  __syncthreads();
  const long long col0 = static_cast<long long>(bg) * nb;
  if (pass == 0) {
    for (int i = threadIdx.x; i < nb; i += blockDim.x)
      if (hist[i]) atomicAdd(&w.col_count[col0 + i], hist[i]);
    return;
  }
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    base[i] = hist[i] ? w.col_off[col0 + i] + atomicAdd(&w.col_fill[col0 + i], hist[i]) : 0u;
    hist[i] = 0u;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < (t1 - t0) * k; x += blockDim.x) {
    const int t = t0 + x / k, slot = x % k;
    const int c = sel[((static_cast<long long>(b) * T + t) * G + g) * k + slot];
    if (c >= 0) {
      const uint32_t pos = base[c] + atomicAdd(&hist[c], 1u);
      w.entries[pos] = (static_cast<uint32_t>(t) << 6) | static_cast<uint32_t>(slot);
    }
  }
}

// Exclusive scans of the column counts (entries) and of their tile counts.
__global__ void __launch_bounds__(1024) scan_columns_kernel(PrefillWs w, int tpt) {
  __shared__ uint32_t warp_a[32], warp_b[32];
  __shared__ uint32_t carry_a, carry_b;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_a = carry_b = 0u;
  __syncthreads();
  for (long long base = 0; base < w.ncol; base += 1024) {
    const long long i = base + threadIdx.x;
    const uint32_t c = i < w.ncol ? w.col_count[i] : 0u;
    const uint32_t tl = (c + tpt - 1) / tpt;
    uint32_t a = c, b = tl;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t ya = __shfl_up_sync(0xffffffffu, a, off);
      const uint32_t yb = __shfl_up_sync(0xffffffffu, b, off);
      if (lane >= off) {
        a += ya;
        b += yb;
      }
    }
    if (lane == 31) {
      warp_a[warp] = a;
      warp_b[warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t sa = warp_a[lane], sb = warp_b[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t ya = __shfl_up_sync(0xffffffffu, sa, off);
        const uint32_t yb = __shfl_up_sync(0xffffffffu, sb, off);
        if (lane >= off) {
          sa += ya;
          sb += yb;
        }
      }
      warp_a[lane] = sa;
      warp_b[lane] = sb;
    }
    __syncthreads();
    const uint32_t pa = (warp ? warp_a[warp - 1] : 0u) + a - c + carry_a;
    const uint32_t pb = (warp ? warp_b[warp - 1] : 0u) + b - tl + carry_b;
    if (i < w.ncol) {
      w.col_off[i] = pa;
      w.tile_off[i] = pb;
    }
    __syncthreads();
    if (threadIdx.x == 1023) {
      carry_a = pa + c;
      carry_b = pb + tl;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    w.col_off[w.ncol] = carry_a;
    w.tile_off[w.ncol] = carry_b;
  }
}

__global__ void make_tiles_kernel(PrefillWs w, int tpt) {
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < w.ncol;
       c += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint32_t n = w.col_count[c];
    const uint32_t t0 = w.tile_off[c], e0 = w.col_off[c];
    for (uint32_t i = 0; i * tpt < n; ++i)
      w.tiles[t0 + i] = make_int4(static_cast<int>(c), static_cast<int>(e0 + i * tpt),
                                  static_cast<int>(min(static_cast<uint32_t>(tpt), n - i * tpt)), 0);
  }
}

// ------------------------------------------------------ 3. KV-outer attention
struct AttnParams {
  PrefillWs w;
  uint32_t* err;
  int T, N, H, G, r, k, nb, q_off, tpt;
  float scale_log2;
};

template <int D>
struct AttnSmem {
  static constexpr uint32_t kKV = 128u * D * 2u;     // one K (or V) block tile
  static constexpr uint32_t kQ = 128u * D * 2u;      // 128 query rows
  static constexpr uint32_t kP = 128u * 128u * 2u;   // P tile (128 rows x 128 keys)
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffV = 2 * kKV;
  static constexpr uint32_t kOffQ = 4 * kKV;
  static constexpr uint32_t kOffP = 4 * kKV + 2 * kQ;
  static constexpr uint32_t kOffBar = kOffP + kP;
  static constexpr uint32_t kBytes = kOffBar + 256;
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    kvouter_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using L = AttnSmem<D>;
  constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
  constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);     // P (K-major) x V (MN-major)
  constexpr uint32_t kTmemCols = 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* kvfull = bars;        // [2]
  uint64_t* kvempty = bars + 2;   // [2]
  uint64_t* qfull = bars + 4;     // [2]
  uint64_t* qempty = bars + 6;    // [2]
  uint64_t* sfull = bars + 8;     // [2]
  uint64_t* sempty = bars + 10;   // [2]
  uint64_t* pfull = bars + 12;    // [1]
  uint64_t* pvdone = bars + 13;   // [1]
  uint64_t* ofree = bars + 14;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long ntiles = static_cast<long long>(p.w.tile_off[p.w.ncol]);
  const long long t_begin = ntiles * blockIdx.x / gridDim.x;
  const long long t_end = ntiles * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kvfull[i], 1);
      mbar_init(&kvempty[i], 1);
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 128);
      mbar_init(&ofree[i], 128);
    }
    mbar_init(pfull, 128);
    mbar_init(pvdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // zero the Q tiles so that rows of absent tokens hold finite values
  for (uint32_t x = threadIdx.x; x < 2 * L::kQ / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[x] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;          // S buffers: columns [0,128) and [128,256)
  const uint32_t tO = tmem + 256;    // O buffers: columns [256, 256+D) and [256+D, 256+2D)

  if (warp == 0) {
    // ----------------------------------------------------------------- TMA
    // The whole warp walks the tiles: lane j gathers tokens j, j+32, ... of a
    // tile, so the entry loads and the per-token Q copies proceed in parallel.
    // Tile descriptors are read two tiles ahead, entries one tile ahead.
    if (t_begin < t_end) {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      const int4 zero4 = make_int4(-1, 0, 0, 0);
      int4 td_cur = p.w.tiles[t_begin];
      int4 td_nx = t_begin + 1 < t_end ? p.w.tiles[t_begin + 1] : zero4;
      uint32_t ent_cur[4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
        ent_cur[x] = lane + 32 * x < td_cur.z ? p.w.entries[td_cur.y + lane + 32 * x] : 0u;
      int prev_col = -1;
      long long u = -1;   // column ordinal
      for (long long ti = t_begin; ti < t_end; ++ti) {
        const long long i = ti - t_begin;
        const int4 td = td_cur;
        uint32_t ent[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) ent[x] = ent_cur[x];
        const int4 td_nn = ti + 2 < t_end ? p.w.tiles[ti + 2] : zero4;
#pragma unroll
        for (int x = 0; x < 4; ++x)
          ent_cur[x] = lane + 32 * x < td_nx.z ? p.w.entries[td_nx.y + lane + 32 * x] : 0u;
        td_cur = td_nx;
        td_nx = td_nn;

        const int col = td.x;
        const int bg = static_cast<int>(col / p.nb);
        const int blk = static_cast<int>(col - static_cast<long long>(bg) * p.nb);
        int ok = 1;
        if (col != prev_col) {
          prev_col = col;
          ++u;
          const int st = static_cast<int>(u & 1);
          if (lane == 0) {
            ok = mbar_wait(&kvempty[st], ((u >> 1) & 1) ^ 1, abort_flag, p.err) ? 1 : 0;
            if (ok) {
              mbar_arrive_expect_tx(&kvfull[st], 2 * L::kKV);
#pragma unroll
              for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(smem + L::kOffK + st * L::kKV + c * 16384, &tm_k, &kvfull[st], c * 64,
                            blk * 128, bg);
                tma_load_3d(smem + L::kOffV + st * L::kKV + c * 16384, &tm_v, &kvfull[st], c * 64,
                            blk * 128, bg);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
        const int qb = static_cast<int>(i & 1);
        const int cnt = td.z;
        if (lane == 0) {
          ok = mbar_wait(&qempty[qb], ((i >> 1) & 1) ^ 1, abort_flag, p.err) ? 1 : 0;
          if (ok) mbar_arrive_expect_tx(&qfull[qb], static_cast<uint32_t>(cnt * p.r * D * 2));
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const int b = bg / p.G, g = bg % p.G;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int j = lane + 32 * x;
          if (j < cnt) {
            const int t = static_cast<int>(ent[x] >> 6);
            const int row = (b * p.T + t) * p.H + g * p.r;
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_2d(smem + L::kOffQ + qb * L::kQ + c * 16384 + j * p.r * 128, &tm_q,
                          &qfull[qb], c * 64, row);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0 && t_begin < t_end) {
      const long long n = t_end - t_begin;
      bool ok = true;
      int prev_col = -1;
      long long u = -1;
      int cur_stage = 0;
      // columns of the next two tiles, read ahead of use
      int col_cur = p.w.tiles[t_begin].x;
      int col_nx = n > 1 ? p.w.tiles[t_begin + 1].x : -1;
      int stage_of[2] = {0, 0};
      bool last_of_col[2] = {false, false};
      auto issue_s = [&](long long i) -> bool {
        const long long ti = t_begin + i;
        const int col = col_cur;
        const int col_next = col_nx;
        col_cur = col_nx;
        col_nx = i + 2 < n ? p.w.tiles[ti + 2].x : -1;
        if (col != prev_col) {
          prev_col = col;
          ++u;
          cur_stage = static_cast<int>(u & 1);
          if (!mbar_wait(&kvfull[cur_stage], (u >> 1) & 1, abort_flag, p.err)) return false;
        }
        const int qb = static_cast<int>(i & 1);
        stage_of[qb] = cur_stage;
        last_of_col[qb] = col_next != col;
        if (!mbar_wait(&qfull[qb], (i >> 1) & 1, abort_flag, p.err)) return false;
        if (!mbar_wait(&sempty[qb], ((i >> 1) & 1) ^ 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + L::kOffQ + qb * L::kQ);
        const uint32_t ka = smem_u32(smem + L::kOffK + cur_stage * L::kKV);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          tc_mma_ss(tS + qb * 128, smem_desc(qa + off, 16, 1024, 2),
                    smem_desc(ka + off, 16, 1024, 2), kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&sfull[qb]);
        tc_commit(&qempty[qb]);
        return true;
      };
      ok = issue_s(0);
      for (long long i = 0; ok && i < n; ++i) {
        const int qb = static_cast<int>(i & 1);
        const int st = stage_of[qb];
        const bool last = last_of_col[qb];
        if (i + 1 < n && !(ok = issue_s(i + 1))) break;
        if (!(ok = mbar_wait(pfull, i & 1, abort_flag, p.err))) break;
        if (!(ok = mbar_wait(&ofree[qb], ((i >> 1) & 1) ^ 1, abort_flag, p.err))) break;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + L::kOffP);
        const uint32_t va = smem_u32(smem + L::kOffV + st * L::kKV);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {   // 128 keys in steps of 16
          const uint64_t ad = smem_desc(pa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(va + ks * 16 * 128, 16384, 1024, 2);
          tc_mma_ss(tO + qb * D, ad, bd, kIdescO, ks > 0 ? 1u : 0u);
        }
        tc_commit(pvdone);
        if (last) tc_commit(&kvempty[st]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tok = row / p.r, head = row % p.r;
    const long long n = t_end - t_begin;
    uint8_t* prow = smem + L::kOffP + row * 128;
    // descriptors two tiles ahead, this row's entry one tile ahead
    const int4 zero4 = make_int4(-1, 0, 0, 0);
    int4 td_cur = n > 0 ? p.w.tiles[t_begin] : zero4;
    int4 td_nx = n > 1 ? p.w.tiles[t_begin + 1] : zero4;
    uint32_t ent_cur = tok < td_cur.z ? p.w.entries[td_cur.y + tok] : 0u;
    // state of the tile whose output is pending
    bool pend_valid = false;
    long long pend_row = 0;     // row of the part arrays: ((b*T + t)*k + slot)*H + h
    float pend_inv_l = 0.f;
    bool ok = true;
    for (long long i = 0; i <= n && ok; ++i) {
      bool cur_valid = false;
      long long cur_row = 0;
      float cur_inv_l = 0.f;
      uint32_t pk[64];
      if (i < n) {
        const int qb = static_cast<int>(i & 1);
        const int4 td = td_cur;
        const uint32_t e = ent_cur;
        const int4 td_nn = i + 2 < n ? p.w.tiles[t_begin + i + 2] : zero4;
        ent_cur = tok < td_nx.z ? p.w.entries[td_nx.y + tok] : 0u;
        td_cur = td_nx;
        td_nx = td_nn;
        const int col = td.x;
        const int bg = static_cast<int>(col / p.nb);
        const int blk = static_cast<int>(col - static_cast<long long>(bg) * p.nb);
        const int b = bg / p.G, g = bg % p.G;
        cur_valid = tok < td.z;
        int lim = 127;
        if (cur_valid) {
          const int t = static_cast<int>(e >> 6), slot = static_cast<int>(e & 63u);
          const int pos = p.q_off + t;
          if ((pos >> 7) == blk) lim = pos & 127;
          cur_row = ((static_cast<long long>(b) * p.T + t) * p.k + slot) * p.H + g * p.r + head;
        }
        if (!(ok = mbar_wait(&sfull[qb], (i >> 1) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + qb * 128 + lane_off + c * 32, sv + c * 32);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&sempty[qb]);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          sv[c] = c <= lim ? sv[c] : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        const float mxs = mx * p.scale_log2;
        float l = 0.f;
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float e0 = fast_exp2(fmaf(sv[c], p.scale_log2, -mxs));
          const float e1 = fast_exp2(fmaf(sv[c + 1], p.scale_log2, -mxs));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
          pk[c >> 1] = *reinterpret_cast<uint32_t*>(&h2);
          const float2 back = __bfloat1622float2(h2);
          l += back.x + back.y;
        }
        cur_inv_l = 1.f / l;
        if (cur_valid) p.w.part_lse[cur_row] = mxs + log2f(l);
      }
      // epilogue of the previous tile (its PV also frees the P buffer)
      if (i > 0) {
        const long long ip = i - 1;
        const int ob = static_cast<int>(ip & 1);
        if (!(ok = mbar_wait(pvdone, ip & 1, abort_flag, p.err))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + ob * D + lane_off + c * 32, ov);
          tc_wait_ld();
          if (pend_valid) {
            uint4* dst = reinterpret_cast<uint4*>(p.w.part_o + pend_row * D + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              __nv_bfloat162 h0 = __floats2bfloat162_rn(ov[8 * x] * pend_inv_l, ov[8 * x + 1] * pend_inv_l);
              __nv_bfloat162 h1 = __floats2bfloat162_rn(ov[8 * x + 2] * pend_inv_l, ov[8 * x + 3] * pend_inv_l);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[8 * x + 4] * pend_inv_l, ov[8 * x + 5] * pend_inv_l);
              __nv_bfloat162 h3 = __floats2bfloat162_rn(ov[8 * x + 6] * pend_inv_l, ov[8 * x + 7] * pend_inv_l);
              dst[x] = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                  *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&ofree[ob]);
      }
      if (i < n) {
        // P row -> shared memory, 128-byte swizzled K-major layout (2 chunks of 64 keys)
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int chunk = u >> 3, unit = u & 7;
          uint4* dst = reinterpret_cast<uint4*>(prow + chunk * 16384 + ((unit ^ (row & 7)) << 4));
          *dst = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(pfull);
        pend_valid = cur_valid;
        pend_row = cur_row;
        pend_inv_l = cur_inv_l;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------- 4. combine
// One CTA per (sequence, token): merge the k normalised partials of each of
// the H heads by their log-sum-exp.  Partials of one token are laid out
// [slot][head][d], so each slot is one contiguous H*d run.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ sel,
                                                      const PrefillWs w, uint16_t* __restrict__ o,
                                                      float* __restrict__ lse, int H, int G,
                                                      int r, int k) {
  constexpr int CH = D / 8;                  // 16-byte chunks per head row
  extern __shared__ float sm_lse[];          // [k][H] log2 units, -inf for unused slots
  const long long bt = blockIdx.x;           // b*T + t
  const float* lsrc = w.part_lse + bt * k * H;
  const int32_t* srow = sel + bt * G * k;
  for (int x = threadIdx.x; x < k * H; x += blockDim.x) {
    const int s = x / H, h = x % H;
    sm_lse[x] = srow[(h / r) * k + s] >= 0 ? lsrc[x] : -INFINITY;
  }
  __syncthreads();
  const uint16_t* osrc = w.part_o + bt * k * H * D;
  for (int item = threadIdx.x; item < H * CH; item += blockDim.x) {
    const int h = item / CH, c = item % CH;
    float M = -INFINITY;
    for (int s = 0; s < k; ++s) M = fmaxf(M, sm_lse[s * H + h]);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float den = 0.f;
#pragma unroll 4
    for (int s = 0; s < k; ++s) {
      const float ls = sm_lse[s * H + h];
      if (ls == -INFINITY) continue;
      const float ws = exp2f(ls - M);
      den += ws;
      const uint4 u = __ldcs(reinterpret_cast<const uint4*>(osrc + (static_cast<long long>(s) * H + h) * D) + c);
      const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wds[e]));
        acc[2 * e] += ws * f.x;
        acc[2 * e + 1] += ws * f.y;
      }
    }
    const float inv = 1.f / den;
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 x = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      out[e] = *reinterpret_cast<uint32_t*>(&x);
    }
    *(reinterpret_cast<uint4*>(o + (bt * H + h) * D) + c) = make_uint4(out[0], out[1], out[2], out[3]);
    if (lse && c == 0) lse[bt * H + h] = (M + log2f(den)) / kLog2e;
  }
}

template <int D>
cudaError_t launch_attn(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const AttnParams& p, const DevCtx* ctx,
                        cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const uint64_t dq[2] = {static_cast<uint64_t>(D),
                          static_cast<uint64_t>(s.batch) * s.seq_q * s.n_q_heads};
  const uint64_t sq[1] = {static_cast<uint64_t>(D) * 2};
  const uint32_t bq[2] = {64, static_cast<uint32_t>(p.r)};
  const uint64_t dk[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(s.seq_kv),
                          static_cast<uint64_t>(s.batch) * s.n_kv_heads};
  const uint64_t sk[2] = {static_cast<uint64_t>(D) * 2,
                          static_cast<uint64_t>(s.seq_kv) * D * 2};
  const uint32_t bk[3] = {64, 128, 1};
  if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = AttnSmem<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(kvouter_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    ProfScope ps_("kvouter_attn", st);
    kvouter_attn_kernel<D><<<ctx->num_sms, kAttnThreads, smem, st>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

}  // namespace

size_t prefill_workspace_bytes(const msa_shape& s) { return carve_bytes(s); }

cudaError_t launch_sparse_prefill(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const int32_t* sel, uint16_t* o,
                                  float* lse, void* ws, cudaStream_t st) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  PrefillWs w = carve(s, ws);
  const int nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  const int r = s.n_q_heads / s.n_kv_heads;
  const int tpt = 128 / r;
  cudaError_t e = cudaMemsetAsync(w.col_count, 0, 4 * w.ncol, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.col_fill, 0, 4 * w.ncol, st);
  if (e != cudaSuccess) return e;
  const dim3 hgrid(static_cast<unsigned>(ceil_div(s.seq_q, kHistTokens)),
                   static_cast<unsigned>(s.batch * s.n_kv_heads));
  const size_t hsmem = 8ull * nb;
  if (hsmem > 200 * 1024) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(sel_invert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(hsmem));
  if (e != cudaSuccess) return e;
  {
    ProfScope ps_("sel_count", st);
    sel_invert_kernel<<<hgrid, 256, hsmem, st>>>(sel, w, s.seq_q, s.n_kv_heads, s.topk, nb, 0);
  }
  {
    ProfScope ps_("scan_columns", st);
    scan_columns_kernel<<<1, 1024, 0, st>>>(w, tpt);
  }
  {
    ProfScope ps_("sel_scatter", st);
    sel_invert_kernel<<<hgrid, 256, hsmem, st>>>(sel, w, s.seq_q, s.n_kv_heads, s.topk, nb, 1);
  }
  {
    ProfScope ps_("make_tiles", st);
    make_tiles_kernel<<<static_cast<unsigned>(ceil_div(w.ncol, 256)), 256, 0, st>>>(w, tpt);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  AttnParams p{};
  p.w = w;
  p.err = ctx->err;
  p.T = s.seq_q;
  p.N = s.seq_kv;
  p.H = s.n_q_heads;
  p.G = s.n_kv_heads;
  p.r = r;
  p.k = s.topk;
  p.nb = nb;
  p.q_off = s.q_offset;
  p.tpt = tpt;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(s.head_dim));
  e = s.head_dim == 128 ? launch_attn<128>(s, q, k, v, p, ctx, st)
                        : launch_attn<64>(s, q, k, v, p, ctx, st);
  if (e != cudaSuccess) return e;
  const unsigned ntok = static_cast<unsigned>(static_cast<long long>(s.batch) * s.seq_q);
  const size_t csmem = sizeof(float) * s.topk * s.n_q_heads;
  {
    ProfScope ps_("combine", st);
    if (s.head_dim == 128)
      combine_kernel<128><<<ntok, 256, csmem, st>>>(sel, w, o, lse, s.n_q_heads, s.n_kv_heads, r,
                                                    s.topk);
    else
      combine_kernel<64><<<ntok, 256, csmem, st>>>(sel, w, o, lse, s.n_q_heads, s.n_kv_heads, r,
                                                   s.topk);
  }
  return cudaGetLastError();
}

}  // namespace msa
