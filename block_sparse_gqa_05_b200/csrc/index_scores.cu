// Index branch scoring with the block max-pool fused in (yhxrc.cn article on
// the MSA figure, section 第一步: one index query per GQA group, one index key
// shared by all heads, score Q_idx . K_idx, block max-pooling).
//
// Prefill: persistent tcgen05 GEMM.  A = 128 (token, group) rows of q_idx,
// B = two 128-key blocks of k_idx, D = 128 x 256 fp32 scores in TMEM.  The
// epilogue masks keys past each row's position and reduces the 128 columns to
// one pooled value, so token scores never leave the SM.
// With the top-k fused in (the whole layer's prefill path), each CTA walks
// whole row tiles over all of their causal key blocks, the epilogue hands each
// block maximum to a top-k warpgroup through a shared-memory ring, and that
// warpgroup keeps every row's running top-(k-1) and writes the selection
// (lumi-systems AI news: the exponential-free top-k; yhxrc.cn 第一步: the index
// branch only has to produce the ordering), so the pooled scores never reach
// memory either.
// Decode (T*G < 128): a bandwidth-bound scan of k_idx with mma.sync.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kStages = 4;       // 256-key k_idx tiles in flight
constexpr int kAcc = 2;          // TMEM accumulator buffers of 256 columns
// warp 0: TMA, warp 1: MMA (warps 2-3 idle), warps 4..11: epilogue, in whole
// warpgroups so that the fused variant can move registers between them
constexpr int kThreads = 384;
constexpr int kTopkThreads = 128;   // fused top-k: warps 12..15, one thread per row
constexpr int kChunkBlocks = 32; // key blocks per work item
constexpr int kRing = 8;         // fused top-k: ring slots of one 256-key tile's two block maxima
// barriers (K stages, Q, accumulators, ring), the TMEM address and the abort
// flag, rounded up; the fused top-k ring follows them
constexpr uint32_t kBarBytes = ((2 * kStages + 4 + 2 * kAcc + 2 * kRing + 1) * 8 + 8 + 127) / 128 * 128;

struct IdxParams {
  float* pooled;
  int32_t* sel;  // fused top-k: [B, T, G, k]
  const int32_t* pages;   // paged index keys: [B, nb] page of each block, or nullptr
  int num_pages;
  uint32_t* err;
  int T, N, G, q_off, nb, k;
  int rowmajor;  // items are whole row tiles, largest first (fused top-k)
  int M;         // row tiles per sequence = ceil(T*G / 128)
  int tpt;       // tokens per row tile = 128 / G
  int kc;        // key blocks per chunk
  int C;         // chunks per sequence
  long long items_per_seq;
  long long items_total;
};

// First row tile whose causal key range reaches chunk c (tiles >= it are valid).
__host__ __device__ inline int chunk_mmin(const IdxParams& p, int c) {
  const long long need = static_cast<long long>(c) * p.kc * 128 - p.q_off + 1;
  long long m = need <= 0 ? 0 : (need + p.tpt - 1) / p.tpt - 1;
  if (m < 0) m = 0;
  if (m > p.M - 1) m = p.M - 1;
  return static_cast<int>(m);
}

// Number of causal key blocks of row tile m (blocks 0 .. ncb-1).
__host__ __device__ inline int tile_causal_blocks(const IdxParams& p, int m) {
  long long t_last = static_cast<long long>(p.tpt) * (m + 1) - 1;
  if (t_last > p.T - 1) t_last = p.T - 1;
  return static_cast<int>((p.q_off + t_last) / 128 + 1);
}

struct ItemCursor {
  int seq = -1, c = 0, cnt = 0;
  long long base = 0;
};

// Work items are ordered (sequence, chunk, row tile); each CTA walks its items
// in increasing order, so the chunk cursor only moves forward.
__device__ inline void item_decode(const IdxParams& p, long long w, ItemCursor& cur, int& seq,
                                   int& m, int& b0, int& b1) {
  if (p.rowmajor) {
    seq = static_cast<int>(w / p.M);
    m = p.M - 1 - static_cast<int>(w - static_cast<long long>(seq) * p.M);
    b0 = 0;
    b1 = tile_causal_blocks(p, m);
    return;
  }
  const int s = static_cast<int>(w / p.items_per_seq);
  const long long r = w - static_cast<long long>(s) * p.items_per_seq;
  if (s != cur.seq) {
    cur.seq = s;
    cur.c = 0;
    cur.base = 0;
    cur.cnt = p.M - chunk_mmin(p, 0);
  }
  while (r >= cur.base + cur.cnt) {
    cur.base += cur.cnt;
    cur.c += 1;
    cur.cnt = p.M - chunk_mmin(p, cur.c);
  }
  seq = s;
  m = chunk_mmin(p, cur.c) + static_cast<int>(r - cur.base);
  b0 = cur.c * p.kc;
  const int ncb = tile_causal_blocks(p, m);
  b1 = min(b0 + p.kc, ncb);
}

// Maximum of 128 scores with three-input max (four chains of 32 values).
MSA_DEV float block_max128(const float* v) {
  float m4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m4[i] = fmax3(v[i], v[i + 4], v[i + 8]);
#pragma unroll
  for (int c = 12; c < 124; c += 8)
#pragma unroll
    for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], v[c + i], v[c + 4 + i]);
#pragma unroll
  for (int i = 0; i < 4; ++i) m4[i] = fmaxf(m4[i], v[124 + i]);
  return fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
}

// KMAX = 0: pooled scores out.  KMAX in {16, 32}: the top-k is fused (k <=
// KMAX) and the selection is written instead; each row keeps the KMAX - 1
// best of its candidate blocks.
template <int DI, int KMAX>
__global__ void __launch_bounds__(kThreads + (KMAX > 0 ? kTopkThreads : 0), 1)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k, const IdxParams p) {
  constexpr uint32_t kQTile = 128u * DI * 2u;       // 128 (token, group) rows
  constexpr uint32_t kKTile = 256u * DI * 2u;       // 256 keys = two blocks
  constexpr uint32_t kLayout = DI == 64 ? 2u : 4u;  // 128-byte / 64-byte swizzle
  constexpr uint32_t kSbo = 8u * DI * 2u;           // 8-row swizzle atom
  constexpr uint32_t kIdesc = idesc_bf16(128, 256, 0, 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qbuf = smem;
  uint8_t* kbuf = smem + 2 * kQTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(kbuf + kStages * kKTile);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + kStages;
  uint64_t* qfull = bars + 2 * kStages;
  uint64_t* qempty = qfull + 2;
  uint64_t* accfull = qempty + 2;
  uint64_t* accempty = accfull + kAcc;
  uint64_t* ring_full = accempty + kAcc;     // fused top-k: [kRing] block maxima written
  uint64_t* ring_empty = ring_full + kRing;  // fused top-k: [kRing] block maxima consumed
  uint64_t* mma_drain = ring_empty + kRing;  // the MMA thread's last commit before exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // fused top-k: [kRing][2 blocks][128 rows] block maxima, after the barriers
  float* ring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1);
    }
    for (int i = 0; i < kAcc; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 128);
    }
    if constexpr (KMAX > 0) {
      for (int i = 0; i < kRing; ++i) {
        mbar_init(&ring_full[i], 128);
        mbar_init(&ring_empty[i], kTopkThreads);
      }
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // fused variant: registers from the producer warpgroup and the top-k
  // warpgroup to the epilogue (which holds a 128-score row)
  constexpr uint32_t kRegEpi = KMAX == 0 ? 0 : (KMAX <= 16 ? 176 : 152);
  constexpr uint32_t kRegTopk = KMAX == 0 ? 0 : (KMAX <= 16 ? 104 : 152);
  static_assert(KMAX == 0 || (56 + 2 * kRegEpi + kRegTopk <= 4 * 128 && kRegEpi > 128),
                "register split of the launch (128 per thread)");
  if (warp < 4) {
    if constexpr (KMAX > 0) regs_dec<56>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      ItemCursor cur;
      long long j = 0, q = 0;   // K tiles and query tiles whose loads were issued
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < p.items_total; w += gridDim.x) {
        int seq, m, b0, b1;
        item_decode(p, w, cur, seq, m, b0, b1);
        const int qb = static_cast<int>(q & 1);
        if (!(ok = mbar_wait(&qempty[qb], ((q >> 1) & 1) ^ 1, abort_flag, p.err))) break;
        mbar_arrive_expect_tx(&qfull[qb], kQTile);
        tma_load_2d(qbuf + qb * kQTile, &tm_q, &qfull[qb], 0, seq * p.T * p.G + m * 128);
        ++q;
        // paged index keys: a 256-key tile is two 128-row pages; a block past
        // the sequence's table loads its last page (those scores are unused).
        // Each tile's page ids are read one tile ahead, so that their latency
        // overlaps the wait for a free stage.
        auto page_row = [&](int blk) -> int {
          const int bb = blk < p.nb ? blk : p.nb - 1;
          return page_of(p.pages, p.nb, p.num_pages, seq, bb, p.err) * 128;
        };
        int pr0 = 0, pr1 = 0;
        if (p.pages && b0 < b1) {
          pr0 = page_row(b0);
          pr1 = page_row(b0 + 1);
        }
        for (int b = b0; b < b1; b += 2) {
          const int s = static_cast<int>(j % kStages);
          if (!(ok = mbar_wait(&kempty[s], ((j / kStages) & 1) ^ 1, abort_flag, p.err))) break;
          mbar_arrive_expect_tx(&kfull[s], kKTile);
          if (p.pages) {
            tma_load_2d(kbuf + s * kKTile, &tm_k, &kfull[s], 0, pr0);
            tma_load_2d(kbuf + s * kKTile + kKTile / 2, &tm_k, &kfull[s], 0, pr1);
            if (b + 2 < b1) {
              pr0 = page_row(b + 2);
              pr1 = page_row(b + 3);
            }
          } else {
            tma_load_2d(kbuf + s * kKTile, &tm_k, &kfull[s], 0, seq * p.N + b * 128);
          }
          ++j;
        }
      }
      // every load issued lands before the CTA may exit
      for (long long t = q > 2 ? q - 2 : 0; t < q; ++t) mbar_drain(&qfull[t & 1], (t >> 1) & 1);
      for (long long t = j > kStages ? j - kStages : 0; t < j; ++t)
        mbar_drain(&kfull[t % kStages], (t / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      ItemCursor cur;
      long long j = 0, q = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < p.items_total; w += gridDim.x, ++q) {
        int seq, m, b0, b1;
        item_decode(p, w, cur, seq, m, b0, b1);
        const int qb = static_cast<int>(q & 1);
        if (!(ok = mbar_wait(&qfull[qb], (q >> 1) & 1, abort_flag, p.err))) break;
        const uint32_t qaddr = smem_u32(qbuf + qb * kQTile);
        for (int b = b0; b < b1; b += 2, ++j) {
          const int s = static_cast<int>(j % kStages);
          const int a = static_cast<int>(j % kAcc);
          if (!(ok = mbar_wait(&kfull[s], (j / kStages) & 1, abort_flag, p.err))) break;
          if (!(ok = mbar_wait(&accempty[a], ((j / kAcc) & 1) ^ 1, abort_flag, p.err))) break;
          tc_fence_after();
          const uint32_t kaddr = smem_u32(kbuf + s * kKTile);
#pragma unroll
          for (int ks = 0; ks < DI / 16; ++ks) {
            const uint64_t ad = smem_desc(qaddr + ks * 32, 16, kSbo, kLayout);
            const uint64_t bd = smem_desc(kaddr + ks * 32, 16, kSbo, kLayout);
            tc_mma_ss(tmem + a * 256, ad, bd, kIdesc, ks > 0 ? 1u : 0u);
          }
          tc_commit(&kempty[s]);
          tc_commit(&accfull[a]);
        }
        if (ok) tc_commit(&qempty[qb]);
      }
      // every MMA issued completes before TMEM is released
      tc_drain(mma_drain, 0);
    }
    __syncwarp();
  }
  } else if (warp < 12) {
    // --------------------------------------------- epilogue: mask + block max
    // Warpgroup wg owns accumulator wg and takes every other 256-key tile;
    // each tile holds two key blocks.
    if constexpr (KMAX > 0) regs_inc<kRegEpi>();
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t taddr_row = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + wg * 256;
    ItemCursor cur;
    long long j = 0;
    bool ok = true;
    const int rows_per_seq = p.T * p.G;
    for (long long w = blockIdx.x; ok && w < p.items_total; w += gridDim.x) {
      int seq, m, b0, b1;
      item_decode(p, w, cur, seq, m, b0, b1);
      const int trow = m * 128 + row;
      const bool valid = trow < rows_per_seq;
      const int t = trow / p.G;
      const int pos = p.q_off + t;
      const int bt = pos >> 7;
      float* out = KMAX > 0 ? nullptr
                            : p.pooled + (static_cast<long long>(seq) * rows_per_seq + trow) *
                                             static_cast<long long>(p.nb);
      for (int b = b0; b < b1; b += 2, ++j) {
        if ((j & 1) != wg) continue;
        if (!(ok = mbar_wait(&accfull[wg], (j >> 1) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        const int slot = static_cast<int>(j % kRing);
        if constexpr (KMAX > 0) {
          // the ring slot must have been consumed by the top-k warpgroup
          if (!(ok = mbar_wait(&ring_empty[slot], ((j / kRing) & 1) ^ 1, abort_flag, p.err)))
            break;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(taddr_row + h * 128 + c * 32, v + c * 32);
          tc_wait_ld();
          if (h == 1) {
            tc_fence_before();
            mbar_arrive(&accempty[wg]);
          }
          const int bb = b + h;
          if constexpr (KMAX > 0) {
            // every candidate block lies below the row's local block, so all
            // of its keys are causal: no mask
            ring[(slot * 2 + h) * 128 + row] = block_max128(v);
          } else if (valid && bb < b1 && bb <= bt) {
            const int lim = (bb == bt) ? (pos & 127) : 127;
            float mx;
            if (lim == 127) {
              mx = block_max128(v);
            } else {
              mx = -INFINITY;
#pragma unroll
              for (int c = 0; c < 128; ++c) mx = fmaxf(mx, c <= lim ? v[c] : -INFINITY);
            }
            out[bb] = mx;
          }
        }
        if constexpr (KMAX > 0) mbar_arrive(&ring_full[slot]);
      }
    }
  } else if constexpr (KMAX > 0) {
    // ------------------------------------------------------- fused top-k
    // Thread t owns row t of every row tile.  Candidate blocks 0 .. b_t - 1
    // arrive in increasing order; the row keeps its KMAX - 1 best as
    // order-preserving score keys, sorted descending.  A block enters only if
    // its key beats the last kept one (strictly: an equal score from a later,
    // higher block loses the tie to the lower block already kept), and it is
    // inserted below every kept key it does not beat.  No exponentials.
    // the launch gives every thread 128 registers: a larger share is an
    // increase, a smaller one a release
    if constexpr (kRegTopk > 128) regs_inc<kRegTopk>();
    else regs_dec<kRegTopk>();
    constexpr int L = KMAX > 1 ? KMAX - 1 : 1;
    const int row = threadIdx.x - kThreads;
    ItemCursor cur;
    long long j = 0;
    bool ok = true;
    const int rows_per_seq = p.T * p.G;
    for (long long w = blockIdx.x; ok && w < p.items_total; w += gridDim.x) {
      int seq, m, b0, b1;
      item_decode(p, w, cur, seq, m, b0, b1);
      const int trow = m * 128 + row;
      const bool valid = trow < rows_per_seq;
      const int bt = (p.q_off + trow / p.G) >> 7;   // the row's local block
      uint32_t tk[L];
      int ti[L];
#pragma unroll
      for (int x = 0; x < L; ++x) {
        tk[x] = 0u;   // below every score key
        ti[x] = 0x7FFFFFFF;
      }
      for (int b = b0; b < b1; b += 2, ++j) {
        const int slot = static_cast<int>(j % kRing);
        if (!(ok = mbar_wait(&ring_full[slot], (j / kRing) & 1, abort_flag, p.err))) break;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int bb = b + h;
          const uint32_t u = float_order_key(ring[(slot * 2 + h) * 128 + row]);
          if (bb < bt && u > tk[L - 1]) {
            bool c[L];
#pragma unroll
            for (int x = 0; x < L; ++x) c[x] = u > tk[x];
#pragma unroll
            for (int x = L - 1; x > 0; --x) {
              tk[x] = c[x - 1] ? tk[x - 1] : (c[x] ? u : tk[x]);
              ti[x] = c[x - 1] ? ti[x - 1] : (c[x] ? bb : ti[x]);
            }
            tk[0] = c[0] ? u : tk[0];
            ti[0] = c[0] ? bb : ti[0];
          }
        }
        mbar_arrive(&ring_empty[slot]);
      }
      if (!ok) break;
      if (!valid) continue;
      // the kk best in ascending block order, then the local block, then -1
      const int kk = min(p.k - 1, bt);
      constexpr int S = L + 1;   // a power of two
      int srt[S];
#pragma unroll
      for (int x = 0; x < S; ++x) srt[x] = x < L && x < kk ? ti[x] : 0x7FFFFFFF;
#pragma unroll
      for (int a = 2; a <= S; a <<= 1)
#pragma unroll
        for (int d = a >> 1; d > 0; d >>= 1)
#pragma unroll
          for (int x = 0; x < S; ++x) {
            const int y = x ^ d;
            if (y > x) {
              const bool up = (x & a) == 0;
              const int lo = min(srt[x], srt[y]), hi = max(srt[x], srt[y]);
              srt[x] = up ? lo : hi;
              srt[y] = up ? hi : lo;
            }
          }
      int32_t* out = p.sel + (static_cast<long long>(seq) * rows_per_seq + trow) * p.k;
#pragma unroll
      for (int x = 0; x < KMAX; ++x)
        if (x < p.k) out[x] = x < kk ? srt[x] : (x == kk ? bt : -1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// pooled[row, b] = -inf for every b > b_t (rows are (seq, t, g)); one warp per row.
__global__ void fill_upper_kernel(float* pooled, long long rows, int T, int G, int q_off,
                                  int nb) {
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int t = static_cast<int>((r / G) % T);
    const int bt = (q_off + t) >> 7;
    float* out = pooled + r * nb;
    for (int b = bt + 1 + (threadIdx.x & 31); b < nb; b += 32) out[b] = -INFINITY;
  }
}

// --------------------------------------------------------------- decode scan
// One CTA per (sequence*T + t, chunk of 8 blocks) (rows on grid.x, which has
// no 65535 limit); warp w owns block 8*chunk+w.  With a page table the 128
// index-key rows of a block are those of its page.
// S[key, group] = k_idx[key, :] . q_idx[t, group, :] on mma.sync m16n8k16 with
// the 16 keys of a tile as rows and 8 groups as columns.  The K dimension is
// permuted identically for both operands so that each thread reads contiguous
// bytes: thread quad q holds index dims [q*4*KS, (q+1)*4*KS), and k-step ks
// uses dims 4*ks .. 4*ks+3 of that range.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int DI>
__global__ void __launch_bounds__(256) index_scores_scan_kernel(const uint16_t* __restrict__ q_idx,
                                                                const uint16_t* __restrict__ k_idx,
                                                                float* __restrict__ pooled, int T,
                                                                int N, int G, int q_off, int nb,
                                                                const int32_t* __restrict__ lens,
                                                                const int32_t* __restrict__ pages,
                                                                int num_pages, uint32_t* err) {
  constexpr int KS = DI / 16;          // k-steps
  constexpr int W = KS * 2;            // 32-bit words per thread per row
  griddep_launch_dependents();         // the top-k may launch (it waits for this kernel)
  const int row_bt = blockIdx.x;       // seq * T + t
  const int seq = row_bt / T;
  const int t = row_bt - seq * T;
  // ragged decode: the query sits at the end of its own cache
  const int pos = lens ? ragged_len(lens, seq, N, err) - 1 : q_off + t;
  const int bt = pos >> 7;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.y * 8 + warp;
  if (blk > bt) return;
  const int gq = lane >> 2, qd = lane & 3;
  // the block's 128 index-key rows (rows past N exist only in a page)
  const uint16_t* kblk =
      pages ? k_idx + static_cast<long long>(page_of(pages, nb, num_pages, seq, blk, err)) * 128 * DI
            : k_idx + (static_cast<long long>(seq) * N + blk * 128) * DI;
  for (int g0 = 0; g0 < G; g0 += 8) {
    // B operand: index query of group g0 + gq, this thread's dim range
    uint32_t bw[W];
    const int grp = g0 + gq;
    if (grp < G) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(
          q_idx + (static_cast<long long>(row_bt) * G + grp) * DI + qd * 4 * KS);
#pragma unroll
      for (int x = 0; x < W; ++x) bw[x] = src[x];
    } else {
#pragma unroll
      for (int x = 0; x < W; ++x) bw[x] = 0u;
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 2
    for (int tile = 0; tile < 8; ++tile) {
      const int key0 = blk * 128 + tile * 16 + gq;
      const int key1 = key0 + 8;
      uint32_t r0[W], r1[W];
      if (key0 < N) {
        const uint4* s0 = reinterpret_cast<const uint4*>(kblk + (tile * 16 + gq) * DI +
                                                         qd * 4 * KS);
#pragma unroll
        for (int x = 0; x < W / 4; ++x) {
          uint4 u = __ldg(s0 + x);
          r0[4 * x] = u.x; r0[4 * x + 1] = u.y; r0[4 * x + 2] = u.z; r0[4 * x + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int x = 0; x < W; ++x) r0[x] = 0u;
      }
      if (key1 < N) {
        const uint4* s1 = reinterpret_cast<const uint4*>(kblk + (tile * 16 + gq + 8) * DI +
                                                         qd * 4 * KS);
#pragma unroll
        for (int x = 0; x < W / 4; ++x) {
          uint4 u = __ldg(s1 + x);
          r1[4 * x] = u.x; r1[4 * x + 1] = u.y; r1[4 * x + 2] = u.z; r1[4 * x + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int x = 0; x < W; ++x) r1[x] = 0u;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t a[4] = {r0[2 * ks], r1[2 * ks], r0[2 * ks + 1], r1[2 * ks + 1]};
        const uint32_t b[2] = {bw[2 * ks], bw[2 * ks + 1]};
        mma_bf16_16816(acc, a, b);
      }
      if (key0 <= pos) {
        mx0 = fmaxf(mx0, acc[0]);
        mx1 = fmaxf(mx1, acc[1]);
      }
      if (key1 <= pos) {
        mx0 = fmaxf(mx0, acc[2]);
        mx1 = fmaxf(mx1, acc[3]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    if (gq == 0) {
      const int ga = g0 + 2 * qd, gb = ga + 1;
      float* out = pooled + static_cast<long long>(row_bt) * G * nb;
      if (ga < G) out[static_cast<long long>(ga) * nb + blk] = mx0;
      if (gb < G) out[static_cast<long long>(gb) * nb + blk] = mx1;
    }
  }
}

// KMAX = 0: pooled scores into ``pooled``; KMAX > 0: the fused top-k writes
// the selection into ``sel`` (k <= KMAX).
template <int DI, int KMAX>
cudaError_t launch_tc(const msa_shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                      float* pooled, int32_t* sel, PageTable pages, const DevCtx* ctx,
                      cudaStream_t st) {
  IdxParams p{};
  p.pooled = pooled;
  p.sel = sel;
  p.pages = pages.table;
  p.num_pages = pages.num_pages;
  p.k = s.topk;
  p.rowmajor = KMAX > 0 ? 1 : 0;
  p.err = ctx->err;
  p.T = s.seq_q;
  p.N = s.seq_kv;
  p.G = s.n_kv_heads;
  p.q_off = s.q_offset;
  p.nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  p.tpt = 128 / p.G;
  p.M = static_cast<int>(ceil_div(static_cast<int64_t>(p.T) * p.G, 128));
  p.kc = kChunkBlocks;
  p.C = static_cast<int>(ceil_div(static_cast<int64_t>(p.q_off) + p.T, p.kc * 128));
  long long per = 0;
  if (KMAX > 0) {
    per = p.M;   // whole row tiles
  } else {
    for (int c = 0; c < p.C; ++c) per += p.M - chunk_mmin(p, c);
  }
  p.items_per_seq = per;
  p.items_total = per * s.batch;

  CUtensorMap tq, tk;
  const uint64_t dq[2] = {static_cast<uint64_t>(DI),
                          static_cast<uint64_t>(s.batch) * s.seq_q * s.n_kv_heads};
  // contiguous keys: [B*N rows][DI], 256-row boxes; paged: [P*128 rows][DI],
  // one 128-row page per box
  const uint64_t dk[2] = {static_cast<uint64_t>(DI),
                          pages.table ? static_cast<uint64_t>(pages.num_pages) * 128
                                      : static_cast<uint64_t>(s.batch) * s.seq_kv};
  const uint64_t stride[1] = {static_cast<uint64_t>(DI) * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(DI), 128};
  const uint32_t kbox[2] = {static_cast<uint32_t>(DI), pages.table ? 128u : 256u};
  const CUtensorMapSwizzle sw =
      DI == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q_idx, dq, stride, box, sw) ||
      !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k_idx, dk, stride, kbox, sw))
    return cudaErrorInvalidValue;

  // alignment slack, operand tiles, barriers, fused top-k ring
  const size_t smem = 1024 + (2 * 128 + kStages * 256) * DI * 2 + kBarBytes +
                      (KMAX > 0 ? kRing * 2 * 128 * 4 : 0);
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc_kernel<DI, KMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long grid = p.items_total < ctx->num_sms ? p.items_total : ctx->num_sms;
  const int threads = kThreads + (KMAX > 0 ? kTopkThreads : 0);
  {
    ProfScope ps_(KMAX > 0 ? "index_topk_tc" : "index_scores_tc", st);
    index_scores_tc_kernel<DI, KMAX><<<static_cast<unsigned>(grid), threads, smem, st>>>(tq, tk, p);
  }
  return cudaGetLastError();
}

// The tensor-core path needs a full 128-row query tile and (contiguous keys)
// a 256-key box; ragged decode always scans.
bool tc_path(const msa_shape& s, bool paged) {
  return static_cast<long long>(s.seq_q) * s.n_kv_heads >= 128 &&
         (paged || static_cast<long long>(s.batch) * s.seq_kv >= 256);
}

}  // namespace

cudaError_t launch_index_scores(const msa_shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                float* pooled, bool fill_upper, cudaStream_t st,
                                const int32_t* lens, PageTable pages) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  const int nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  const long long rows = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads;
  cudaError_t e;
  if (lens || !tc_path(s, pages.table != nullptr)) {
    const int last_bt = (s.q_offset + s.seq_q - 1) / 128;
    const dim3 grid(static_cast<unsigned>(s.batch * s.seq_q),
                    static_cast<unsigned>(ceil_div(last_bt + 1, 8)));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    ProfScope ps_("index_scores_scan", st);
    if (s.index_dim == 64)
      index_scores_scan_kernel<64><<<grid, 256, 0, st>>>(q_idx, k_idx, pooled, s.seq_q, s.seq_kv,
                                                         s.n_kv_heads, s.q_offset, nb, lens,
                                                         pages.table, pages.num_pages, ctx->err);
    else
      index_scores_scan_kernel<32><<<grid, 256, 0, st>>>(q_idx, k_idx, pooled, s.seq_q, s.seq_kv,
                                                         s.n_kv_heads, s.q_offset, nb, lens,
                                                         pages.table, pages.num_pages, ctx->err);
    e = cudaGetLastError();
  } else {
    e = s.index_dim == 64 ? launch_tc<64, 0>(s, q_idx, k_idx, pooled, nullptr, pages, ctx, st)
                          : launch_tc<32, 0>(s, q_idx, k_idx, pooled, nullptr, pages, ctx, st);
  }
  if (e != cudaSuccess || !fill_upper) return e;
  const long long warps_needed = rows;
  long long blocks = (warps_needed + 7) / 8;
  if (blocks > 65535LL * 8) blocks = 65535LL * 8;
  {
    ProfScope ps_("fill_upper", st);
    fill_upper_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(pooled, rows, s.seq_q,
                                                                   s.n_kv_heads, s.q_offset, nb);
  }
  return cudaGetLastError();
}

// Whole row tiles are the fused kernel's work items.  Few, long ones (the
// 1M-context chunk: 512 row tiles of 8192 blocks each) leave the persistent
// grid's CTAs with uneven shares, and there the chunked kernel plus the
// standalone top-k is faster; many row tiles, or short rows, balance.  The
// rule depends on the shape alone, so workspace sizes do not depend on the
// device.
bool index_topk_fusable(const msa_shape& s, bool paged) {
  if (!tc_path(s, paged) || s.topk > 32) return false;
  const long long row_tiles = static_cast<long long>(s.batch) *
                              ceil_div(static_cast<int64_t>(s.seq_q) * s.n_kv_heads, 128);
  return row_tiles >= 1024 || ceil_div(s.seq_kv, 128) <= 1024;
}

cudaError_t launch_index_topk(const msa_shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                              int32_t* sel, cudaStream_t st, PageTable pages) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  if (!index_topk_fusable(s, pages.table != nullptr)) return cudaErrorNotSupported;
  if (s.topk <= 16)
    return s.index_dim == 64 ? launch_tc<64, 16>(s, q_idx, k_idx, nullptr, sel, pages, ctx, st)
                             : launch_tc<32, 16>(s, q_idx, k_idx, nullptr, sel, pages, ctx, st);
  return s.index_dim == 64 ? launch_tc<64, 32>(s, q_idx, k_idx, nullptr, sel, pages, ctx, st)
                           : launch_tc<32, 32>(s, q_idx, k_idx, nullptr, sel, pages, ctx, st);
}

}  // namespace msa

namespace msa {
cudaError_t set_wait_limit_index(uint64_t ns) { return set_wait_limit_here(ns); }
}  // namespace msa
