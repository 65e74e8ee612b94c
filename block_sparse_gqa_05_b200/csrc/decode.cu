// Decode attention (one query token per sequence), sparse (MSA main branch:
// yhxrc.cn article, section 第二步; lumi-systems AI news: exact block-sparse
// attention over the selected blocks) and dense causal GQA (the baseline).
//
// Work items are (sequence, group, block) visits: the k selected blocks of a
// (sequence, group) for sparse decode, all of its causal blocks for dense
// decode.  A persistent grid of one CTA per SM takes a contiguous range of
// items; one TMA warp streams the K and V tiles of its blocks (128-byte
// swizzle) through a ring of stages while eight consumer warps compute.
// The heads of a group are the 16 rows of mma.sync m16n8k16 tiles
// (zero-padded when r < 16): for Q K^T each warp owns 16 keys of the block,
// the row maxima and sums are exchanged through shared memory, P is staged
// there in bf16, and for P V each warp owns D/8 output columns, so no
// per-warp state has to be merged at the end.  A (sequence, group) whose
// items all fall in one CTA is written directly; one that spans CTAs leaves
// a normalised partial per CTA, merged by the last CTA to finish it (chosen
// by an atomic counter: no CTA ever waits for another).  The kernel is bound
// by HBM bandwidth on the K/V bytes.  With a page table the K/V tile of
// logical block j of a sequence is read from that block's page.
#include <math.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;   // 8 consumer warps + 1 TMA warp
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxGrid = 256;
constexpr int kMergeOnePass = 8;   // most CTAs a (sequence, group) may span for the one-pass merge
constexpr int kPStride = 136;    // bf16 per row of the P tile: rows 272 B apart, no bank conflicts
constexpr float kLog2e = 1.4426950408889634f;

struct DecParams {
  const uint16_t* q;      // [B, 1, H, d]
  const int32_t* sel;     // [B, 1, G, k] (sparse) or nullptr (dense)
  const int32_t* lens;    // [B] cache lengths (ragged decode) or nullptr: all N
  const int32_t* pages;   // [B, nb] page of each logical block, or nullptr (contiguous)
  int num_pages, nb;
  uint16_t* o;            // [B, 1, H, d]
  float* lse;             // [B, 1, H] or nullptr
  uint32_t* counters;     // [B*G] CTAs done with a (sequence, group)
  float* part_lse;        // [2*grid, r]   (log2 units)
  float* part_o;          // [2*grid, r, d] normalised partial outputs
  uint32_t* err;
  long long n_items;      // B*G*per_bg
  int per_bg;             // items of one (sequence, group): k, or the causal blocks
  int N, H, G, r, k;
  float scale_log2;
};

template <int D>
struct DecLayout {
  static constexpr uint32_t kTile = 128u * D * 2u;             // K (or V) of one block
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr uint32_t kOffP = kStages * 2u * kTile;      // P [16][kPStride] bf16
  static constexpr uint32_t kOffRed = kOffP + 16u * kPStride * 2u;   // wmax, wsum [8][16]
  static constexpr uint32_t kOffBar = kOffRed + 2u * 8u * 16u * 4u;
  static constexpr uint32_t kOffFlag = kOffBar + 3u * kStages * 8u;  // abort, last[2]
  static constexpr uint32_t kBytes = kOffFlag + 16u;
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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
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

// Query position of sequence b: the last row of its cache.
__device__ __forceinline__ int query_pos(const DecParams& p, int b) {
  return p.lens ? ragged_len(p.lens, b, p.N, p.err) - 1 : p.N - 1;
}

// Block of item i (-1 when it has nothing to attend to: an empty selection
// slot or a block past the query), and its (sequence, group) in *bg.
__device__ __forceinline__ int item_block(const DecParams& p, long long i, int* bg) {
  const int g = static_cast<int>(i / p.per_bg);
  const int j = static_cast<int>(i - static_cast<long long>(g) * p.per_bg);
  *bg = g;
  const int bt = query_pos(p, g / p.G) >> 7;
  const int blk = p.sel ? __ldg(p.sel + static_cast<long long>(g) * p.k + j) : j;
  return (blk >= 0 && blk <= bt) ? blk : -1;
}

// First item of CTA c, and the CTA holding item i (ranges split evenly).
__device__ __forceinline__ long long cta_first(long long c, long long n, long long grid) {
  return c * n / grid;
}
__device__ __forceinline__ int cta_of(long long i, long long n, long long grid) {
  return static_cast<int>(((i + 1) * grid + n - 1) / n - 1);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  using L = DecLayout<D>;
  constexpr int S = L::kStages;
  constexpr int KS = D / 16;          // k-steps of Q K^T
  constexpr int NW = D / 64;          // n8 tiles of P V per warp (D/8 columns)
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* ps = reinterpret_cast<uint16_t*>(smem + L::kOffP);
  float* wmax = reinterpret_cast<float*>(smem + L::kOffRed);
  float* wsum = wmax + 8 * 16;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* vfull = kfull + S;
  uint64_t* empty = vfull + S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffFlag);
  volatile int* s_last = abort_flag + 1;   // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n = p.n_items, grid = gridDim.x;
  const long long i0 = cta_first(blockIdx.x, n, grid);
  const long long i1 = cta_first(blockIdx.x + 1, n, grid);

  // the swizzled K/V tiles need 1024-byte alignment; the launch reserves no slack
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrTimeout);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // this kernel may start while the one before it (the top-k) finishes: the
  // selection is read only after it is complete
  griddep_wait();
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    int cnt = 0;
    bool ok = true;
    for (long long base = i0; ok && base < i1; base += 32) {
      int bgv = 0;
      const int blk = base + lane < i1 ? item_block(p, base + lane, &bgv) : -1;
      // TMA coordinates of the block's rows: (row, sequence*G + group) in a
      // contiguous cache, (0, page*G + group) in a paged one
      int yv = 0, zv = 0;
      if (blk >= 0) {
        if (p.pages) {
          zv = page_of(p.pages, p.nb, p.num_pages, bgv / p.G, blk, p.err) * p.G + bgv % p.G;
        } else {
          yv = blk * 128;
          zv = bgv;
        }
      }
      unsigned m = __ballot_sync(0xffffffffu, blk >= 0);
      while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1;
        const int y_ = __shfl_sync(0xffffffffu, yv, src);
        const int z_ = __shfl_sync(0xffffffffu, zv, src);
        const int s = cnt % S;
        if (lane == 0) {
          ok = mbar_wait(&empty[s], ((cnt / S) & 1) ^ 1, abort_flag, p.err);
          if (ok) {
            mbar_arrive_expect_tx(&kfull[s], L::kTile);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + s * 2 * L::kTile + c * 16384, &tm_k, &kfull[s], c * 64, y_, z_);
            mbar_arrive_expect_tx(&vfull[s], L::kTile);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + s * 2 * L::kTile + L::kTile + c * 16384, &tm_v, &vfull[s],
                          c * 64, y_, z_);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
        ++cnt;
      }
    }
    // Every load this warp issued lands before the CTA may exit.
    if (lane == 0) {
      for (int x = max(0, cnt - S); x < cnt; ++x) {
        const int s = x % S;
        const uint32_t ph = (x / S) & 1;
        const uint64_t t0 = globaltimer();
        while (!(mbar_test(&kfull[s], ph) && mbar_test(&vfull[s], ph)))
          if (globaltimer() - t0 > kDrainLimitNs) {
            atomicOr(p.err, kErrTimeout);
            break;
          }
      }
    }
    return;
  }

  // ---------------------------------------------------------- consumer warps
  const int w = warp;
  const int gq = lane >> 2, qd = lane & 3;
  const uint32_t pbase = smem_u32(ps);
  int cnt = 0;
  int cur_bg = -1;
  int pos = 0;                     // query position of the current sequence
  long long seg_first = 0;
  bool failed = false;
  uint32_t qa[KS][4];
  float m_run[2], l_run[2];
  float o_acc[NW][4];

  // Partials of this CTA still to be announced: the group whose items open
  // its range (slot 0) and the one whose items close it (slot 1).
  int pend[2] = {-1, -1};

  // Write the (sequence, group) just finished: directly when this CTA holds
  // all of its items, else as a normalised partial in this CTA's slot.
  auto finish = [&](int bg, long long first, long long end) {
    const int b = bg / p.G, g = bg % p.G;
    const int r = p.r;
    float inv[2], lse2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      inv[h] = l_run[h] > 0.f ? 1.f / l_run[h] : 0.f;
      lse2[h] = l_run[h] > 0.f ? m_run[h] + log2f(l_run[h]) : -INFINITY;
    }
    const long long bfirst = static_cast<long long>(bg) * p.per_bg;
    if (first == bfirst && end == bfirst + p.per_bg) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = gq + 8 * h;
        if (row >= r) continue;
        uint16_t* orow = p.o + (static_cast<long long>(b) * p.H + g * r + row) * D;
#pragma unroll
        for (int nt = 0; nt < NW; ++nt) {
          const int col = w * (D / 8) + nt * 8 + 2 * qd;
          *reinterpret_cast<uint32_t*>(orow + col) =
              pack_bf16(o_acc[nt][2 * h] * inv[h], o_acc[nt][2 * h + 1] * inv[h]);
        }
        if (p.lse && w == 0 && qd == 0)
          p.lse[static_cast<long long>(b) * p.H + g * r + row] = lse2[h] / kLog2e;
      }
      return;
    }
    const int which = first == i0 ? 0 : 1;
    pend[which] = bg;
    const int slot = 2 * static_cast<int>(blockIdx.x) + which;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = gq + 8 * h;
      if (row >= r) continue;
      float* prow = p.part_o + (static_cast<long long>(slot) * r + row) * D;
#pragma unroll
      for (int nt = 0; nt < NW; ++nt) {
        const int col = w * (D / 8) + nt * 8 + 2 * qd;
        *reinterpret_cast<float2*>(prow + col) =
            make_float2(o_acc[nt][2 * h] * inv[h], o_acc[nt][2 * h + 1] * inv[h]);
      }
      if (w == 0 && qd == 0) p.part_lse[static_cast<long long>(slot) * r + row] = lse2[h];
    }
  };

  for (long long base = i0; !failed && base < i1; base += 32) {
    int bgv = 0;
    const int blkv = base + lane < i1 ? item_block(p, base + lane, &bgv) : -1;
    const int nin = static_cast<int>(min(32LL, i1 - base));
    for (int jj = 0; jj < nin; ++jj) {
      const int blk = __shfl_sync(0xffffffffu, blkv, jj);
      const int bg = __shfl_sync(0xffffffffu, bgv, jj);
      if (bg != cur_bg) {
        if (cur_bg >= 0) finish(cur_bg, seg_first, base + jj);
        cur_bg = bg;
        pos = query_pos(p, bg / p.G);
        seg_first = base + jj;
        const int b = bg / p.G, g = bg % p.G;
        const uint16_t* qb = p.q + (static_cast<long long>(b) * p.H + g * p.r) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int c0 = ks * 16 + 2 * qd;
          qa[ks][0] = gq < p.r ? __ldg(reinterpret_cast<const uint32_t*>(qb + gq * D + c0)) : 0u;
          qa[ks][1] =
              gq + 8 < p.r ? __ldg(reinterpret_cast<const uint32_t*>(qb + (gq + 8) * D + c0)) : 0u;
          qa[ks][2] =
              gq < p.r ? __ldg(reinterpret_cast<const uint32_t*>(qb + gq * D + c0 + 8)) : 0u;
          qa[ks][3] = gq + 8 < p.r
                          ? __ldg(reinterpret_cast<const uint32_t*>(qb + (gq + 8) * D + c0 + 8))
                          : 0u;
        }
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
#pragma unroll
        for (int nt = 0; nt < NW; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) o_acc[nt][e] = 0.f;
      }
      if (blk < 0) continue;
      const int s = cnt % S;
      const uint32_t ph = (cnt / S) & 1;
      ++cnt;
      const uint32_t kbase = smem_u32(smem + s * 2 * L::kTile);
      const uint32_t vbase = kbase + L::kTile;

      // ---- S = Q K^T for keys w*16 .. w*16+15 of the block
      const bool okk = mbar_wait(&kfull[s], ph, abort_flag, p.err);
      float sv[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = w * 16 + nt * 8 + gq;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t bb[2];
          const int col = ks * 16 + 2 * qd;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(bb[0]) : "r"(kbase + sw128_off(key, col)));
          asm volatile("ld.shared.b32 %0, [%1];"
                       : "=r"(bb[1])
                       : "r"(kbase + sw128_off(key, col + 8)));
          mma16816(sv[nt], qa[ks], bb);
        }
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = blk * 128 + w * 16 + nt * 8 + 2 * qd + (e & 1);
          sv[nt][e] = key <= pos ? sv[nt][e] * p.scale_log2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], sv[nt][e]);
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      }
      if (qd == 0) {
        wmax[w * 16 + gq] = mx[0];
        wmax[w * 16 + gq + 8] = mx[1];
      }
      if (named_bar_or(1, kConsumerThreads, !okk || *abort_flag)) {
        failed = true;
        *abort_flag = 1;
        break;
      }
      // ---- block row maxima, P = exp2(S - m) in bf16, row sums
      float corr[2], mnew[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float bm = -INFINITY;
#pragma unroll
        for (int x = 0; x < 8; ++x) bm = fmaxf(bm, wmax[x * 16 + gq + 8 * h]);
        mnew[h] = fmaxf(m_run[h], bm);
        corr[h] = mnew[h] == -INFINITY ? 1.f : exp2f(m_run[h] - mnew[h]);
        m_run[h] = mnew[h];
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mh = mnew[e >> 1];
          const float pv = mh == -INFINITY ? 0.f : exp2f(sv[nt][e] - mh);
          sv[nt][e] = pv;
          rs[e >> 1] += pv;
        }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = w * 16 + nt * 8 + 2 * qd;
        *reinterpret_cast<uint32_t*>(ps + gq * kPStride + key) = pack_bf16(sv[nt][0], sv[nt][1]);
        *reinterpret_cast<uint32_t*>(ps + (gq + 8) * kPStride + key) =
            pack_bf16(sv[nt][2], sv[nt][3]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
        rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
      }
      if (qd == 0) {
        wsum[w * 16 + gq] = rs[0];
        wsum[w * 16 + gq + 8] = rs[1];
      }
      const bool okv = mbar_wait(&vfull[s], ph, abort_flag, p.err);
      if (named_bar_or(1, kConsumerThreads, !okv || *abort_flag)) {
        failed = true;
        *abort_flag = 1;
        break;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float bs = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) bs += wsum[x * 16 + gq + 8 * h];
        l_run[h] = l_run[h] * corr[h] + bs;
      }
#pragma unroll
      for (int nt = 0; nt < NW; ++nt) {
        o_acc[nt][0] *= corr[0];
        o_acc[nt][1] *= corr[0];
        o_acc[nt][2] *= corr[1];
        o_acc[nt][3] *= corr[1];
      }
      // ---- O[:, w*D/8 ..] += P V over the block's 128 keys.  Keys past the
      // query have P = 0, but their V rows can hold anything (a ragged cache
      // past its length), and 0 * NaN is NaN: in the block that holds the
      // query, those rows are zeroed in the B fragments.  Register j of a
      // fragment holds keys ks*16 + 8*(j&1) + 2*qd + {0 (low half), 1}.
      const int mi = lane >> 3, ri = lane & 7;
      const bool past_query = blk * 128 + 127 > pos;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t pa[4];
        ldsm_x4(pbase + static_cast<uint32_t>(((mi & 1) * 8 + ri) * kPStride * 2 +
                                              (ks * 16 + (mi >> 1) * 8) * 2),
                pa);
        const int vkey = ks * 16 + (mi & 1) * 8 + ri;
        uint32_t vb[2 * NW];
        if constexpr (NW == 2)
          ldsm_x4_trans(vbase + sw128_off(vkey, w * 16 + (mi >> 1) * 8), vb);
        else
          ldsm_x2_trans(vbase + sw128_off(vkey, w * 8), vb);
        if (past_query) {
#pragma unroll
          for (int j = 0; j < 2 * NW; ++j) {
            const int k0 = blk * 128 + ks * 16 + 8 * (j & 1) + 2 * qd;
            vb[j] &= (k0 <= pos ? 0x0000FFFFu : 0u) | (k0 + 1 <= pos ? 0xFFFF0000u : 0u);
          }
        }
        mma16816(o_acc[0], pa, vb);
        if constexpr (NW == 2) mma16816(o_acc[1], pa, vb + 2);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  if (failed) return;
  if (cur_bg >= 0) finish(cur_bg, seg_first, i1);
  if (pend[0] < 0 && pend[1] < 0) return;

  // Announce the partials; the last CTA to finish a group merges its
  // partials.  Every load of the ring has been consumed, so the stage memory
  // holds the merge weights.
  __threadfence();
  named_bar_sync(1, kConsumerThreads);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      s_last[x] = 0;
      if (pend[x] < 0) continue;
      const long long bfirst = static_cast<long long>(pend[x]) * p.per_bg;
      const int cf = cta_of(bfirst, n, grid), cl = cta_of(bfirst + p.per_bg - 1, n, grid);
      const uint32_t prev = atomicAdd(&p.counters[pend[x]], 1u);
      s_last[x] = prev == static_cast<uint32_t>(cl - cf) ? 1 : 0;
    }
  }
  named_bar_sync(1, kConsumerThreads);
  const int r = p.r;
  float* wgt = reinterpret_cast<float*>(smem);   // [CTAs of the group][r]
#pragma unroll 1
  for (int x = 0; x < 2; ++x) {
    if (!s_last[x]) continue;
    __threadfence();
    const int bg = pend[x];
    const int b = bg / p.G, g = bg % p.G;
    const long long bfirst = static_cast<long long>(bg) * p.per_bg;
    const int cf = cta_of(bfirst, n, grid), cl = cta_of(bfirst + p.per_bg - 1, n, grid);
    const int nc = cl - cf + 1;
    const int sf = 2 * cf + (bfirst == cta_first(cf, n, grid) ? 0 : 1);
    if (nc <= kMergeOnePass) {
      // one pass: each thread loads every partial's log-sum-exp and its four
      // output columns together, so the merge costs one round trip
      for (int e = threadIdx.x; e < r * D / 4; e += kConsumerThreads) {
        const int row = (e * 4) / D, col = (e * 4) % D;
        float lj[kMergeOnePass];
        float4 v4[kMergeOnePass];
#pragma unroll
        for (int c = 0; c < kMergeOnePass; ++c) {
          if (c < nc) {
            const int sl = c == 0 ? sf : 2 * (cf + c);
            lj[c] = __ldcg(&p.part_lse[static_cast<long long>(sl) * r + row]);
            v4[c] = __ldcg(reinterpret_cast<const float4*>(
                p.part_o + (static_cast<long long>(sl) * r + row) * D + col));
          }
        }
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < kMergeOnePass; ++c)
          if (c < nc) M = fmaxf(M, lj[c]);
        float den = 0.f;
#pragma unroll
        for (int c = 0; c < kMergeOnePass; ++c)
          if (c < nc && lj[c] != -INFINITY) den += exp2f(lj[c] - M);
        const float rden = den > 0.f ? 1.f / den : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kMergeOnePass; ++c) {
          if (c < nc && lj[c] != -INFINITY) {
            const float wj = exp2f(lj[c] - M) * rden;
            acc.x += wj * v4[c].x;
            acc.y += wj * v4[c].y;
            acc.z += wj * v4[c].z;
            acc.w += wj * v4[c].w;
          }
        }
        uint2 pk;
        pk.x = pack_bf16(acc.x, acc.y);
        pk.y = pack_bf16(acc.z, acc.w);
        *reinterpret_cast<uint2*>(p.o + (static_cast<long long>(b) * p.H + g * r + row) * D +
                                  col) = pk;
        if (p.lse && col == 0)
          p.lse[static_cast<long long>(b) * p.H + g * r + row] =
              den > 0.f ? (M + log2f(den)) / kLog2e : -INFINITY;
      }
      if (threadIdx.x == 0) p.counters[bg] = 0u;
      named_bar_sync(1, kConsumerThreads);
      continue;
    }
    for (int e = threadIdx.x; e < nc * r; e += kConsumerThreads) {
      const int c = cf + e / r;
      const int sl = c == cf ? sf : 2 * c;
      wgt[e] = __ldcg(&p.part_lse[static_cast<long long>(sl) * r + e % r]);
    }
    named_bar_sync(1, kConsumerThreads);
    // per row: max and sum of the partial weights (warp w: rows w, w + 8)
    for (int row = w; row < r; row += kConsumerWarps) {
      float M = -INFINITY;
      for (int c = lane; c < nc; c += 32) M = fmaxf(M, wgt[c * r + row]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      float den = 0.f;
      for (int c = lane; c < nc; c += 32) {
        const float lj = wgt[c * r + row];
        den += lj == -INFINITY ? 0.f : exp2f(lj - M);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      __syncwarp();
      const float rden = den > 0.f ? 1.f / den : 0.f;
      for (int c = lane; c < nc; c += 32) {
        const float lj = wgt[c * r + row];
        wgt[c * r + row] = lj == -INFINITY ? 0.f : exp2f(lj - M) * rden;
      }
      if (p.lse && lane == 0)
        p.lse[static_cast<long long>(b) * p.H + g * r + row] =
            den > 0.f ? (M + log2f(den)) / kLog2e : -INFINITY;
    }
    named_bar_sync(1, kConsumerThreads);
    // outputs, four columns per thread, every partial's load in flight at once
    for (int e = threadIdx.x; e < r * D / 4; e += kConsumerThreads) {
      const int row = (e * 4) / D, col = (e * 4) % D;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int c = cf; c <= cl; ++c) {
        const int sl = c == cf ? sf : 2 * c;
        const float wj = wgt[(c - cf) * r + row];
        const float4 v4 = __ldcg(reinterpret_cast<const float4*>(
            p.part_o + (static_cast<long long>(sl) * r + row) * D + col));
        acc.x += wj * v4.x;
        acc.y += wj * v4.y;
        acc.z += wj * v4.z;
        acc.w += wj * v4.w;
      }
      uint2 pk;
      pk.x = pack_bf16(acc.x, acc.y);
      pk.y = pack_bf16(acc.z, acc.w);
      *reinterpret_cast<uint2*>(p.o + (static_cast<long long>(b) * p.H + g * r + row) * D + col) =
          pk;
    }
    if (threadIdx.x == 0) p.counters[bg] = 0u;
    named_bar_sync(1, kConsumerThreads);
  }
}

}  // namespace

size_t decode_workspace_bytes(const msa_shape& s, bool dense) {
  const int r = s.n_q_heads / s.n_kv_heads;
  const size_t bg = static_cast<size_t>(s.batch) * s.n_kv_heads;
  const size_t per_bg = dense ? static_cast<size_t>(ceil_div(s.seq_kv, 128))
                              : static_cast<size_t>(s.topk);
  const size_t slots = 2 * std::min(bg * per_bg, static_cast<size_t>(kMaxGrid));
  return align_up(bg * 4, 256) + align_up(slots * r * 4, 256) +
         align_up(slots * r * s.head_dim * 4, 256);
}

cudaError_t prepare_decode(const msa_shape& s, void* ws, cudaStream_t st) {
  const size_t bg = static_cast<size_t>(s.batch) * s.n_kv_heads;
  return cudaMemsetAsync(ws, 0, bg * 4, st);   // the counters open the workspace
}

cudaError_t launch_decode(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* sel, uint16_t* o, float* lse,
                          void* ws, bool dense, cudaStream_t st, const int32_t* lens,
                          PageTable pages, bool counters_zeroed) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  const int r = s.n_q_heads / s.n_kv_heads;
  const size_t bg = static_cast<size_t>(s.batch) * s.n_kv_heads;
  const int per_bg = dense ? static_cast<int>(ceil_div(s.seq_kv, 128)) : s.topk;
  const long long n_items = static_cast<long long>(bg) * per_bg;
  const long long grid = std::min<long long>(
      n_items, std::min<long long>(std::max(ctx->num_sms, 1), kMaxGrid));
  const size_t slots = 2 * static_cast<size_t>(std::min<long long>(n_items, kMaxGrid));
  DecParams p{};
  char* w = static_cast<char*>(ws);
  p.counters = reinterpret_cast<uint32_t*>(w);
  p.part_lse = reinterpret_cast<float*>(w + align_up(bg * 4, 256));
  p.part_o = reinterpret_cast<float*>(w + align_up(bg * 4, 256) + align_up(slots * r * 4, 256));
  p.q = q;
  p.sel = dense ? nullptr : sel;
  p.lens = lens;
  p.pages = pages.table;
  p.num_pages = pages.num_pages;
  p.nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  p.o = o;
  p.lse = lse;
  p.err = ctx->err;
  p.n_items = n_items;
  p.per_bg = per_bg;
  p.N = s.seq_kv;
  p.H = s.n_q_heads;
  p.G = s.n_kv_heads;
  p.r = r;
  p.k = s.topk;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(s.head_dim));
  if (n_items == 0) return cudaSuccess;

  CUtensorMap tk, tv;
  // contiguous: [B*G][N][d]; paged: [num_pages*G][128][d]
  const uint64_t rows = pages.table ? 128 : static_cast<uint64_t>(s.seq_kv);
  const uint64_t mats = pages.table ? static_cast<uint64_t>(pages.num_pages) * s.n_kv_heads : bg;
  const uint64_t dims[3] = {static_cast<uint64_t>(s.head_dim), rows, mats};
  const uint64_t strides[2] = {static_cast<uint64_t>(s.head_dim) * 2,
                               rows * s.head_dim * 2};
  const uint32_t box[3] = {64, 128, 1};
  if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  cudaError_t e = counters_zeroed ? cudaSuccess : cudaMemsetAsync(p.counters, 0, bg * 4, st);
  if (e != cudaSuccess) return e;
  const unsigned g = static_cast<unsigned>(grid);
  if (s.head_dim == 128) {
    const size_t smem = DecLayout<128>::kBytes;
    e = cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    ProfScope ps_("decode_attn", st);
    e = launch_dependent(decode_attn_kernel<128>, dim3(g), dim3(kThreads), smem, st, tk, tv, p);
    if (e != cudaSuccess) return e;
  } else {
    const size_t smem = DecLayout<64>::kBytes;
    e = cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    ProfScope ps_("decode_attn", st);
    e = launch_dependent(decode_attn_kernel<64>, dim3(g), dim3(kThreads), smem, st, tk, tv, p);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace msa

// ------------------------------------------------ decode without allocation
// Split-K scratch of msa_sparse_attn_decode_static: one static array in
// device memory, shared by every call on a device.  Host code only ever
// passes its device address, looked up once per device and cached for the
// life of the process (like the error word: a device reset makes it stale).
namespace msa {
namespace {

static __device__ __align__(256) unsigned char g_decode_static_scratch[MSA_DECODE_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on error).
void* static_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
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
  msa::ApiRange nvtx_("msa_sparse_attn_decode_static");
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

namespace msa {
cudaError_t set_wait_limit_decode(uint64_t ns) { return set_wait_limit_here(ns); }
}  // namespace msa
