// Main branch, prefill: exact softmax attention over the selected blocks
// (yhxrc.cn article, section 第二步: Q/K/V keep the GQA shapes, only the blocks
// listed in I_g are read, every head of group g shares I_g; lumi-systems AI
// news: exact block-sparse attention with a "KV-outer" loop so the tensor
// cores work at block granularity).
//
// Schedule (KV-outer):
//  1. invert sel: for every (sequence, group, block) column, the list of
//     (token, slot) pairs that selected it (counting sort in three passes);
//  2. cut every column into tiles of 128/r tokens = 128 (token, head) rows and
//     deal the tiles of every (sequence, group) segment evenly over the CTAs,
//     segment after segment, so that every CTA gets the same share of every
//     group's work (one contiguous chunk per CTA and segment, the chunks
//     rotated from segment to segment: see plan_ctas_kernel);
//  3. persistent tcgen05 kernel: each selected K/V block is TMA-loaded once per
//     CTA that works on it and reused by every tile of its column; for a tile,
//     S = Q K^T (TMEM), softmax over the block (causal mask on the local
//     block), P (bf16, written back into TMEM), O_part = P V (TMEM) -> bf16
//     partial plus its (max, sum) per (token, slot, head), stored in the order
//     of the column-sorted entry list, so a full tile's partials are one
//     contiguous block (two TMA stores);
//  4. combine the k partials of every (token, head), found through the
//     position of each (token, group, slot) in the entry list.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAttnThreads = 512;   // 4 warpgroups: TMA+MMA, 2 softmax, epilogue
constexpr int kHistTokens = 1024;   // tokens per CTA of the inversion passes

constexpr int kMaxAttnGrid = 1024;  // most CTAs of the attention kernel (one per SM)
struct PrefillWs {
  uint32_t* col_count;   // [ncol]
  uint32_t* col_fill;    // [ncol]
  uint32_t* col_off;     // [ncol + 1]
  uint32_t* tile_off;    // [ncol + 1]  tiles of the columns in column order
  uint32_t* entries;     // [B*T*G*k]   (t << 6) | slot, sorted by column
  uint32_t* inv;         // [B*T*G*k]   position in entries of each selected (t, g, slot)
  uint32_t* cta_off;     // [kMaxAttnGrid + 1] first tile of each CTA in the dealt order
  uint32_t* seg_prefix;  // [nseg * kMaxAttnGrid] tiles of a CTA in the segments before one
  int4* tiles;           // [max_tiles] (column, entry start, count, 0), dealt order
  uint32_t* tile_ent;    // [max_tiles * tpt] entries of each tile, 0xFFFFFFFF past its count
  uint16_t* part_o;      // [entry, r, d] bf16 partial outputs, normalised by their own l
  float* part_ml;        // [entry, r, 2] (running max m, sum l) of each partial, log2 units
  // columns are (b * G + g) * nb + block; a segment is the nb columns of one
  // (b, g)
  long long ncol, nseg, max_tiles;
  size_t bytes;
};

PrefillWs carve(const msa_shape& s, void* base) {
  PrefillWs w{};
  const long long nb = ceil_div(s.seq_kv, 128);
  const int r = s.n_q_heads / s.n_kv_heads;
  const int tpt = 128 / r;
  w.nseg = static_cast<long long>(s.batch) * s.n_kv_heads;
  w.ncol = w.nseg * nb;
  const long long nent = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads * s.topk;
  w.max_tiles = ceil_div(nent, tpt) + std::min(w.ncol, nent);
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
  w.inv = reinterpret_cast<uint32_t*>(take(4 * nent));
  w.cta_off = reinterpret_cast<uint32_t*>(take(4 * (kMaxAttnGrid + 1)));
  w.seg_prefix = reinterpret_cast<uint32_t*>(take(4ull * w.nseg * kMaxAttnGrid));
  w.tiles = reinterpret_cast<int4*>(take(16 * w.max_tiles));
  w.tile_ent = reinterpret_cast<uint32_t*>(take(4ull * w.max_tiles * tpt));
  w.part_o = reinterpret_cast<uint16_t*>(take(2ull * s.batch * s.seq_q * s.n_q_heads *
                                              s.topk * s.head_dim));
  w.part_ml = reinterpret_cast<float*>(take(8ull * s.batch * s.seq_q * s.n_q_heads * s.topk));
  w.bytes = off;
  return w;
}

size_t carve_bytes(const msa_shape& s) { return carve(s, nullptr).bytes; }

// ------------------------------------------------------- 1. invert selection
// grid: (ceil(T / kHistTokens), B*G).  Pass 0 counts (sequence, group, block)
// hits; pass 1 reserves a range per column and scatters (token, slot) entries.
// Only entries 0 <= block <= b_t take part (negative ones are empty slots);
// one past the query's block is ignored, and pass 0 flags it in the error
// word, so a bad caller selection can never index past the histogram.
__global__ void __launch_bounds__(256) sel_invert_kernel(const int32_t* __restrict__ sel,
                                                         PrefillWs w, int T, int G, int k,
                                                         int nb, int q_off, int pass,
                                                         uint32_t* err) {
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
    if (c >= 0 && c <= (q_off + t) >> 7)
      atomicAdd(&hist[c], 1u);
    else if (c >= 0 && pass == 0)
      atomicOr(err, kErrBadSel);
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
    if (c >= 0 && c <= (q_off + t) >> 7) {
      const uint32_t pos = base[c] + atomicAdd(&hist[c], 1u);
      w.entries[pos] = (static_cast<uint32_t>(t) << 6) | static_cast<uint32_t>(slot);
      w.inv[((static_cast<long long>(b) * T + t) * G + g) * k + slot] = pos;
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

// Segment s's n_s tiles, in column order, are cut into grid chunks,
// chunk j = [first(j), first(j + 1)), first(j) = j * n_s / grid; chunk_of(x)
// is the chunk holding segment tile x.  Chunk j goes to CTA (j - s * rot)
// mod grid: the last chunks of a segment (its latest blocks: short columns,
// so more K/V loads per tile, and causally masked tiles) land on a
// different CTA for every segment instead of all on the last CTA.
__device__ __forceinline__ long long deal_first(long long j, long long n, int grid) {
  return j * n / grid;
}
__device__ __forceinline__ int chunk_of(long long x, long long n, int grid) {
  return static_cast<int>(((x + 1) * grid + n - 1) / n - 1);
}
__device__ __forceinline__ int chunk_of_cta(int c, long long sg, int rot, int grid) {
  return static_cast<int>((c + sg * rot) % grid);
}

// One CTA: per attention CTA c, the tiles it holds in the segments before
// each segment (seg_prefix) and its first tile in the dealt order (cta_off).
__global__ void __launch_bounds__(1024) plan_ctas_kernel(PrefillWs w, int nb, int grid, int rot) {
  __shared__ uint32_t warp_sum[32];
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  uint32_t acc = 0;
  if (c < grid) {
    for (long long sg = 0; sg < w.nseg; ++sg) {
      const long long lo = w.tile_off[sg * nb];
      const long long n = static_cast<long long>(w.tile_off[(sg + 1) * nb]) - lo;
      w.seg_prefix[sg * grid + c] = acc;
      const int j = chunk_of_cta(c, sg, rot, grid);
      acc += static_cast<uint32_t>(deal_first(j + 1, n, grid) - deal_first(j, n, grid));
    }
  }
  uint32_t incl = acc;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = warp_sum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    warp_sum[lane] = v;
  }
  __syncthreads();
  const uint32_t excl = (warp ? warp_sum[warp - 1] : 0u) + incl - acc;
  if (c < grid) w.cta_off[c] = excl;
  if (c == grid - 1) w.cta_off[grid] = excl + acc;
}

// One thread per tile: find its column (upper bound in the tile offsets),
// write the descriptor and the tile's entries padded to tpt at the tile's
// place in the dealt order.
__global__ void make_tiles_kernel(PrefillWs w, int tpt, int nb, int grid, int rot) {
  const long long ntiles = static_cast<long long>(w.tile_off[w.ncol]);
  for (long long ti = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; ti < ntiles;
       ti += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long lo = 0, hi = w.ncol;   // first column whose tile offset exceeds ti
    while (lo < hi) {
      const long long mid = (lo + hi) >> 1;
      if (static_cast<long long>(w.tile_off[mid]) > ti) hi = mid; else lo = mid + 1;
    }
    const long long c = lo - 1;
    const uint32_t i = static_cast<uint32_t>(ti - w.tile_off[c]);
    const uint32_t start = w.col_off[c] + i * tpt;
    const uint32_t cnt = min(static_cast<uint32_t>(tpt), w.col_count[c] - i * tpt);
    const long long sg = c / nb;
    const long long slo = w.tile_off[sg * nb];
    const long long n = static_cast<long long>(w.tile_off[(sg + 1) * nb]) - slo;
    const long long x = ti - slo;
    const int j = chunk_of(x, n, grid);
    const int cta = static_cast<int>(((j - sg * rot) % grid + grid) % grid);
    const long long dst = static_cast<long long>(w.cta_off[cta]) + w.seg_prefix[sg * grid + cta] +
                          (x - deal_first(j, n, grid));
    w.tiles[dst] = make_int4(static_cast<int>(c), static_cast<int>(start), static_cast<int>(cnt), 0);
    for (int j = 0; j < tpt; ++j)
      w.tile_ent[dst * tpt + j] = j < static_cast<int>(cnt) ? w.entries[start + j] : 0xFFFFFFFFu;
  }
}

// ------------------------------------------------------ 3. KV-outer attention
struct AttnParams {
  PrefillWs w;
  uint32_t* err;
  int T, N, H, G, r, k, nb, q_off, tpt;
  int q3d;   // r = 8, d = 128: one 3-D TMA load per token ([half][head][64] in smem)
  const int32_t* pages;   // paged K/V: [B, nb] page of each block, or nullptr
  int num_pages;
  float scale_log2;
};

constexpr int kNS = 2;        // S/P buffers in TMEM (128 columns each), one per softmax warpgroup
constexpr int kNO = 2;        // O buffers in TMEM (D columns each), one per softmax warpgroup
constexpr int kMBMax = 16;    // most tiles per metadata batch (two batches in flight)
constexpr int kTentWords = 256; // entry words in the metadata ring (both batches)

template <int D>
struct AttnSmem {
  static constexpr int kNQ = D == 128 ? 2 : 3;   // query tile buffers
  // V tiles: with two, the next column's V loads while this one's PVs run
  static constexpr int kNV = 2;
  static constexpr uint32_t kKV = 128u * D * 2u;     // one K (or V) block tile
  static constexpr uint32_t kQ = 128u * D * 2u;      // 128 query rows
  static constexpr uint32_t kOffK = 0;                      // two K stages
  static constexpr uint32_t kOffV = 2 * kKV;                // kNV V stages
  static constexpr uint32_t kOffQ = kOffV + kNV * kKV;
  // epilogue staging: 128 rows x 64 columns (the rows' halves go out in turn)
  static constexpr uint32_t kOffStage = kOffQ + kNQ * kQ;
  // softmax exchange: float [2 tile parities][2 warpgroups][128 rows] partial
  // row maxima, then the same for the partial row sums
  static constexpr uint32_t kOffXmax = kOffStage + 16384;
  static constexpr uint32_t kOffXsum = kOffXmax + 2048;
  static constexpr uint32_t kOffMeta = kOffXsum + 2048;     // int [kNQ][4] (kNQ <= 4)
  // int4 [2*kMBMax] per tile: group (b*G+g), block, entries, flags (1: first
  // tile of its column here, 2: last)
  static constexpr uint32_t kOffThdr = kOffMeta + 64;
  static constexpr uint32_t kOffTrow = kOffThdr + 2 * kMBMax * 16;   // int [kTentWords] query row
  static constexpr uint32_t kOffBar = kOffTrow + kTentWords * 4;
  // barriers: K 2+2, V kNV+kNV, Q kNQ+kNQ, S/P kNS+kNS, O 2+2, row sums 2+2,
  // metadata 2+2; then the TMEM address and the abort flag
  // + MMA drain + one per V stage for the loads of a paged cache's last block
  static constexpr uint32_t kNBars = 4 + 2 * kNV + 2 * kNQ + 2 * kNS + 12 + 1 + kNV;
  static constexpr uint32_t kBytes = kOffBar + kNBars * 8 + 8;
  static_assert(kBytes <= 227u * 1024u, "shared memory of one CTA");
};

// Roles by warpgroup: WG0 = warps 0 and 3 gather the query tiles (TMA) and
// load K (warp 0) and V (warp 3) at column changes, warp 1 issues the MMAs,
// warp 2 prepares tile metadata; WG1 and WG2 = softmax, both on every tile
// (warpgroup wg takes key columns [64 wg, 64 wg + 64) of each row); WG3 =
// epilogue.  Register budget per thread is moved from WG0/WG3 to the softmax
// warpgroups so that a softmax thread holds its 64 scores.
// TMEM: kNS = 2 S/P buffers of 128 columns, by tile parity (P is written over
// the first 64 columns of its tile's S as packed bf16 and consumed from there
// by the PV MMA), and kNO = 2 O buffers of D columns, so a tile's PV never
// waits for the previous tile's output to be drained: the epilogue has a
// whole tile of time to read O out.  S(j + 2) reuses tile j's buffer and is
// issued once PV(j) is (tcgen05 MMAs of one thread run in issue order).
template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    kvouter_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o,
                        const __grid_constant__ CUtensorMap tm_ot, const AttnParams p) {
  using L = AttnSmem<D>;
  constexpr int kNQ = L::kNQ;
  constexpr int kNV = L::kNV;
  static_assert(kNQ <= 4, "meta holds four query buffers");
  constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
  constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);     // P (TMEM) x V (MN-major)
  constexpr uint32_t kTmemCols = 512;
  static_assert(kNS * 128 + kNO * D <= static_cast<int>(kTmemCols), "TMEM columns");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled operand tiles need 1024-byte alignment; the launch reserves no slack
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  const int kmb = min(kMBMax, (kTentWords / 2) / p.tpt);   // tiles per metadata batch
  float* xmax = reinterpret_cast<float*>(smem + L::kOffXmax);
  float* xsum = reinterpret_cast<float*>(smem + L::kOffXsum);
  int* meta = reinterpret_cast<int*>(smem + L::kOffMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* kfull = bars;               // [2]  K stage loaded
  uint64_t* kempty = bars + 2;          // [2]  K stage free (last S of its column done)
  uint64_t* vfull = bars + 4;           // [kNV] V stage loaded
  uint64_t* vempty = vfull + kNV;       // [kNV] V stage free (last PV of its column done)
  uint64_t* qfull = vempty + kNV;       // [kNQ]
  uint64_t* qempty = qfull + kNQ;       // [kNQ]
  uint64_t* sfull = qempty + kNQ;       // [kNS]
  uint64_t* pfull = sfull + kNS;        // [kNS]
  uint64_t* ofull = pfull + kNS;        // [kNO]
  uint64_t* ofree = ofull + 2;          // [kNO]
  uint64_t* lfull = ofree + 2;          // [2] by tile parity: partial row sums written
  uint64_t* lempty = lfull + 2;         // [2] by tile parity: partial row sums read
  uint64_t* mfull = lempty + 2;         // [2] metadata batch ready
  uint64_t* mempty = mfull + 2;         // [2] metadata batch consumed
  uint64_t* mma_drain = mempty + 2;     // the MMA thread's last commit before exit
  uint64_t* vtail = mma_drain + 1;      // [kNV] V of a paged cache's last block loaded
  int4* thdr = reinterpret_cast<int4*>(smem + L::kOffThdr);
  int* trow = reinterpret_cast<int*>(smem + L::kOffTrow);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(vtail + kNV);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wgid = warp >> 2;
  const long long ntiles = static_cast<long long>(p.w.tile_off[p.w.ncol]);
  const long long t_begin = p.w.cta_off[blockIdx.x];
  const long long t_end = p.w.cta_off[blockIdx.x + 1];
  const long long n = t_end - t_begin;
  const int tpt = p.tpt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&ofull[i], 1);
      mbar_init(&ofree[i], 128);
      mbar_init(&lfull[i], 256);
      mbar_init(&lempty[i], 128);
      mbar_init(&mfull[i], 32);
      mbar_init(&mempty[i], 2);          // both gather warps
    }
    for (int i = 0; i < kNV; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(&qfull[i], 2);           // both gather warps (expect_tx arrivals)
      mbar_init(&qempty[i], 1);
    }
    mbar_init(mma_drain, 1);
    for (int i = 0; i < kNV; ++i) mbar_init(&vtail[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // zero the Q tiles so that rows of absent tokens hold finite values
  for (uint32_t x = threadIdx.x; x < kNQ * L::kQ / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[x] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;                // kNS S/P buffers of 128 columns
  const uint32_t tO = tmem + kNS * 128;    // kNO O buffers of D columns

  if (wgid == 0) {
    regs_dec<64>();
    if (warp == 0 || warp == 3) {
      // ------------------------------------------------------- query gather
      // Warps 0 and 3 walk the tiles together and split every tile's tokens
      // (token j goes to warp j & 1): one TMA request from one thread moves
      // slowly, so two warps issue in parallel.  At a column change warp 0
      // also loads the column's K and warp 3 its V.  Tile metadata comes from
      // the shared ring filled by warp 2.
      const int gw = warp == 0 ? 0 : 1;
      if (n > 0) {
        if (lane == 0) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(gw == 0 ? &tm_k : &tm_v);
        }
        int u = -1;                    // column ordinal
        int ib = 0, ms = 0;            // tile within its metadata batch, batch slot
        uint32_t mph = 0;              // parity of that slot's barriers
        int qb = 0;                    // query buffer
        uint32_t qph = 0;              // its parity
        long long q_armed = 0;         // query tiles this warp issued loads for (lane 0)
        int kv_armed = 0;              // K (warp 0) or V (warp 3) columns loaded (lane 0)
        uint32_t vtail_ph = 0;         // warp 3: parity of each V stage's tail barrier
        const int nx = (tpt + 63) >> 6;   // this warp's tokens per lane (<= 2)
        for (long long i = 0; i < n; ++i) {
          int ok = 1;
          if (ib == 0) {
            ok = mbar_wait(&mfull[ms], mph, abort_flag, p.err) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
          }
          const int4 hd = thdr[ms * kMBMax + ib];
          const int* tr = trow + (ms * kmb + ib) * tpt;
          // this warp's tokens j = 2 * (lane + 32 x) + gw
          int rows[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int j = 2 * (lane + 32 * x) + gw;
            rows[x] = x < nx && j < tpt ? tr[j] : -1;
          }
          __syncwarp();
          if (++ib == kmb || i + 1 == n) {
            if (lane == 0) mbar_arrive(&mempty[ms]);
            ib = 0;
            ms ^= 1;
            if (ms == 0) mph ^= 1u;
          }
          const bool newcol = (hd.w & 1) != 0;
          if (newcol) ++u;
          // the tile's queries first: they never wait on a K or V stage, and
          // S(i) may be needed before the PV that frees the next column's V
          if (lane == 0) {
            ok = mbar_wait(&qempty[qb], qph ^ 1u, abort_flag, p.err) ? 1 : 0;
            if (ok) {
              if (gw == 0) {
                meta[qb * 4 + 0] = u & 1;
                meta[qb * 4 + 1] = newcol ? 1 : 0;
                meta[qb * 4 + 2] = (hd.w & 2) != 0 ? 1 : 0;
              }
              // this warp's tokens of the tile's hd.z
              const int mine = (hd.z + 1 - gw) >> 1;
              mbar_arrive_expect_tx(&qfull[qb], static_cast<uint32_t>(mine * p.r * D * 2));
              ++q_armed;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          uint8_t* qdst = smem + L::kOffQ + qb * L::kQ;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int j = 2 * (lane + 32 * x) + gw;
            if (rows[x] >= 0) {
              if (p.q3d) {
                // token j's 8 heads x 128 columns as [half][head][64]: two 1 KB
                // swizzle atoms, 8-row groups 2 KB apart
                tma_load_3d(qdst + j * 2048, &tm_q, &qfull[qb], 0, rows[x], 0);
              } else {
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                  tma_load_2d(qdst + c * 16384 + j * p.r * 128, &tm_q, &qfull[qb], c * 64,
                              rows[x]);
              }
            }
          }
          // then the column's K (warp 0: stage u % 2 is free once the last S
          // of column u - 2 is done) or V (warp 3: stage u % kNV is free once
          // the last PV of column u - kNV is done)
          if (newcol) {
            if (lane == 0) {
              if (gw == 0) {
                const int st = u & 1;
                ok = mbar_wait(&kempty[st], ((u >> 1) & 1) ^ 1, abort_flag, p.err) ? 1 : 0;
                if (ok) {
                  ++kv_armed;
                  mbar_arrive_expect_tx(&kfull[st], L::kKV);
#pragma unroll
                  for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(smem + L::kOffK + st * L::kKV + c * 16384, &tm_k, &kfull[st],
                                c * 64, hd.y, hd.x);
                }
              } else {
                const int vs = u % kNV;
                ok = mbar_wait(&vempty[vs], ((u / kNV) & 1) ^ 1, abort_flag, p.err) ? 1 : 0;
                if (ok) {
                  // the last block of a paged sequence lands on its own barrier
                  // and reaches the PV through the zeroing below
                  uint64_t* vb = (hd.w & 4) ? &vtail[vs] : &vfull[vs];
                  ++kv_armed;
                  mbar_arrive_expect_tx(vb, L::kKV);
#pragma unroll
                  for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(smem + L::kOffV + vs * L::kKV + c * 16384, &tm_v, vb, c * 64,
                                hd.y, hd.x);
                }
              }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (gw == 1 && (hd.w & 4)) {
              // V rows at or past N: zero them (a weight of 0 times NaN is NaN)
              const int vs = u % kNV;
              const uint32_t ph = (vtail_ph >> vs) & 1u;
              if (lane == 0) ok = mbar_wait(&vtail[vs], ph, abort_flag, p.err) ? 1 : 0;
              ok = __shfl_sync(0xffffffffu, ok, 0);
              vtail_ph ^= 1u << vs;
              if (!ok) {
                // the load lands before the CTA may exit; the stage's full
                // barrier completes so that the drain below finds it done
                if (lane == 0) {
                  mbar_drain(&vtail[vs], ph);
                  mbar_arrive(&vfull[vs]);
                }
                break;
              }
              const int valid = p.N & 127;
              uint8_t* vt = smem + L::kOffV + vs * L::kKV;
              for (int x = lane; x < (128 - valid) * (D / 8); x += 32) {
                const int row = valid + x / (D / 8), unit = x % (D / 8);
                *reinterpret_cast<uint4*>(vt + (unit >> 3) * 16384 + row * 128 + (unit & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(&vfull[vs]);
            }
          }
          if (++qb == kNQ) {
            qb = 0;
            qph ^= 1u;
          }
        }
        // every load this warp issued lands before the CTA may exit
        if (lane == 0) {
          for (long long t = q_armed > kNQ ? q_armed - kNQ : 0; t < q_armed; ++t)
            mbar_drain(&qfull[t % kNQ], (t / kNQ) & 1);
          if (gw == 0) {
            for (int c = kv_armed > 2 ? kv_armed - 2 : 0; c < kv_armed; ++c)
              mbar_drain(&kfull[c & 1], (c >> 1) & 1);
          } else {
            for (int c = kv_armed > kNV ? kv_armed - kNV : 0; c < kv_armed; ++c)
              mbar_drain(&vfull[c % kNV], (c / kNV) & 1);
          }
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ---------------------------------------------------------- metadata
      // Batches of kmb tiles into the shared ring: a header per tile (group,
      // block, entries, first/last tile of its column) and the query row of
      // every token, all loads of a batch in flight together.
      const int tshift = __ffs(tpt) - 1;   // tpt = 128 / r is a power of two
      int pcol = -1;                       // column of the previous batch's last tile
      for (long long bi = 0; bi * kmb < n; ++bi) {
        const int ms = static_cast<int>(bi & 1);
        if (!mbar_wait(&mempty[ms], ((bi >> 1) & 1) ^ 1, abort_flag, p.err)) break;
        const long long a = t_begin + bi * kmb;
        const int nt = static_cast<int>(min(static_cast<long long>(kmb), t_end - a));
        // the batch's tiles and, in lane nt, the tile after it (for its column)
        int4 td = make_int4(-1, 0, 0, 0);
        if (lane <= nt && a + lane < ntiles) td = p.w.tiles[a + lane];
        const int col = td.x;
        const int nextcol = __shfl_down_sync(0xffffffffu, col, 1);
        int prvcol = __shfl_up_sync(0xffffffffu, col, 1);
        if (lane == 0) prvcol = pcol;
        const int bg = col >= 0 ? col / p.nb : 0;
        const int b = bg / p.G, g = bg - b * p.G;
        const int rowbase = b * p.T * p.H + g * p.r;
        if (lane < nt) {
          const int blk = col - bg * p.nb;
          // the K/V TMA coordinates of the column's block: (row, matrix) in
          // [B*G][N][d], or (0, page*G + g) in a paged [P*G][128][d]; flag 4:
          // the block is the last of a paged sequence, whose rows past N may
          // hold any bits and are zeroed in V before the PV
          int z = bg, y = blk * 128, tail = 0;
          if (p.pages) {
            z = page_of(p.pages, p.nb, p.num_pages, b, blk, p.err) * p.G + g;
            y = 0;
            tail = (blk == p.nb - 1 && (p.N & 127) != 0) ? 4 : 0;
          }
          const int flags = (col != prvcol ? 1 : 0) |
                            ((a + lane + 1 >= t_end || nextcol != col) ? 2 : 0) | tail;
          thdr[ms * kMBMax + lane] = make_int4(z, y, td.z, flags);
        }
        // entries of tiles a .. a+nt-1 are contiguous: nt * tpt words
        const int nent = nt * tpt;
        for (int base = 0; base < nent; base += 8 * 32) {
          uint32_t ev[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int idx = base + lane + 32 * x;
            ev[x] = idx < nent ? p.w.tile_ent[a * tpt + idx] : 0xFFFFFFFFu;
          }
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int idx = base + lane + 32 * x;
            const int rb = __shfl_sync(0xffffffffu, rowbase, min(idx >> tshift, 31));
            if (idx < nent)
              trow[(ms * kmb) * tpt + idx] =
                  ev[x] != 0xFFFFFFFFu ? rb + static_cast<int>(ev[x] >> 6) * p.H : -1;
          }
        }
        pcol = __shfl_sync(0xffffffffu, col, nt - 1);
        __syncwarp();
        mbar_arrive(&mfull[ms]);
      }
      __syncwarp();
    } else if (warp == 1) {
      // --------------------------------------------------------------- MMA
      // Two in-order streams, S(j) = Q K^T and PV(i) = P V, issued by one
      // thread as soon as each is ready (polling), so a query gather that is
      // late never holds back the PV of an earlier tile.  S(j) reuses the S/P
      // buffer of tile j-kNS, so it is issued only after PV(j-kNS); tcgen05 MMAs
      // of one thread execute in issue order, which makes that reuse safe.
      if (lane == 0 && n > 0) {
        const bool q3d = p.q3d != 0;
        // descriptors of the operand buffers; a K step adds its byte offset / 16
        const uint64_t dq0 = smem_desc(smem_u32(smem + L::kOffQ), 16, q3d ? 2048 : 1024, 2);
        const uint64_t dk0 = smem_desc(smem_u32(smem + L::kOffK), 16, 1024, 2);
        const uint64_t dv0 = smem_desc(smem_u32(smem + L::kOffV), 16384, 1024, 2);
        long long ns = 0, np = 0;   // next S, next PV
        long long u = -1;           // K column ordinal (S side)
        long long uv = -1;          // V column ordinal (PV side)
        bool last_of_col[4] = {false, false, false, false};
        bool first_of_col[4] = {false, false, false, false};
        bool s_meta = false;        // meta of S(ns) read, waiting for its K stage
        int s_st = 0;
        bool s_last = false;
        uint64_t t_idle = 0;
        while (np < n) {
          bool progress = false;
          // ---- S(ns)
          if (ns < n && ns < np + kNS) {
            const int qb = static_cast<int>(ns % kNQ);
            if (!s_meta && mbar_test(&qfull[qb], (ns / kNQ) & 1)) {
              s_st = meta[qb * 4 + 0];
              const bool newcol = meta[qb * 4 + 1] != 0;
              s_last = meta[qb * 4 + 2] != 0;
              last_of_col[ns & 3] = s_last;
              first_of_col[ns & 3] = newcol;
              if (newcol) ++u;
              s_meta = true;
              s_st |= newcol ? 0x100 : 0;
            }
            if (s_meta && (!(s_st & 0x100) || mbar_test(&kfull[s_st & 1], (u >> 1) & 1))) {
              const int st = s_st & 1;
              tc_fence_after();
              const int sb = static_cast<int>(ns % kNS);
              const uint64_t dq = dq0 + (qb * L::kQ >> 4);
              const uint64_t dk = dk0 + (st * L::kKV >> 4);
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t qoff = q3d ? (ks >> 2) * 1024 + (ks & 3) * 32 : off;
                tc_mma_ss(tS + sb * 128, dq + (qoff >> 4), dk + (off >> 4), kIdescS,
                          ks > 0 ? 1u : 0u);
              }
              tc_commit(&sfull[sb]);
              tc_commit(&qempty[qb]);
              if (s_last) tc_commit(&kempty[st]);
              s_meta = false;
              ++ns;
              progress = true;
            }
          }
          // ---- PV(np)
          if (np < ns) {
            const int sb = static_cast<int>(np % kNS);
            const int ob = static_cast<int>(np % kNO);
            const bool need_v = first_of_col[np & 3];
            const long long un = need_v ? uv + 1 : uv;   // V column of PV(np)
            if ((!need_v || mbar_test(&vfull[un % kNV], (un / kNV) & 1)) &&
                mbar_test(&pfull[sb], (np / kNS) & 1) &&
                mbar_test(&ofree[ob], ((np / kNO) & 1) ^ 1)) {
              uv = un;
              tc_fence_after();
              const uint64_t dv = dv0 + ((uv % kNV) * L::kKV >> 4);
#pragma unroll
              for (int ks = 0; ks < 8; ++ks)   // 128 keys in steps of 16 (8 packed columns)
                tc_mma_ts(tO + ob * D, tS + sb * 128 + ks * 8, dv + (ks * 16 * 128 >> 4), kIdescO,
                          ks > 0 ? 1u : 0u);
              tc_commit(&ofull[ob]);
              if (last_of_col[np & 3]) tc_commit(&vempty[uv % kNV]);
              ++np;
              progress = true;
            }
          }
          if (progress) {
            t_idle = 0;
          } else if (*abort_flag) {
            break;
          } else if (t_idle == 0) {
            t_idle = globaltimer();
          } else if (globaltimer() - t_idle > g_wait_limit_ns) {
            atomicOr(p.err, kErrTimeout);
            *abort_flag = 1;
            break;
          }
        }
        // every MMA issued completes before TMEM is released
        tc_drain(mma_drain, 0);
      }
      __syncwarp();
    }
  } else if (wgid <= 2) {
    // ------------------------------------------- softmax (two warpgroups)
    // Both warpgroups work on every tile: warpgroup wg takes the 64 columns
    // [64 wg, 64 wg + 64) of each row (a warp reaches its quarter's 32 TMEM
    // lanes), which halves a tile's softmax latency, the link of the
    // S -> softmax -> PV chain that paces the kernel.  The two halves'
    // row maxima meet in shared memory (a named barrier over both
    // warpgroups, which also orders every S load before any P store over
    // those columns), and the partial row sums go to the epilogue, which adds
    // them and normalises.
    regs_inc<176>();
    const int wg = wgid - 1;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t sbase = tS + lane_off;
    const int tok = row / p.r, head = row % p.r;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    // the next tile's descriptor and entry are loaded one tile ahead: their
    // latency would otherwise sit between S and the mask of every tile
    int2 cs_next = make_int2(0, 0);
    uint32_t e_next = 0xFFFFFFFFu;
    if (n > 0) {
      cs_next = *reinterpret_cast<const int2*>(&p.w.tiles[t_begin]);
      e_next = tok < tpt ? p.w.tile_ent[t_begin * tpt + tok] : 0xFFFFFFFFu;
    }
    // A role that gives up on a wait (an expired bound) must not leave its
    // partner warpgroup in a named barrier: every exit is decided together,
    // at the barrier, from this tile's waits and the previous tile's.
    bool failed = false;
    for (long long i = 0; i < n; ++i) {
      const int2 cs = cs_next;   // column, entry start
      const uint32_t e = e_next;
      if (i + 1 < n) {
        const long long tn = t_begin + i + 1;
        cs_next = *reinterpret_cast<const int2*>(&p.w.tiles[tn]);
        e_next = tok < tpt ? p.w.tile_ent[tn * tpt + tok] : 0xFFFFFFFFu;
      }
      const int col = cs.x;
      const int sb = static_cast<int>(i % kNS);
      const int par = static_cast<int>(i & 1);
      const uint32_t sbuf = sbase + sb * 128;
      const bool ok = !failed && mbar_wait(&sfull[sb], (i / kNS) & 1, abort_flag, p.err);
      tc_fence_after();
      float sv[64];
      if (ok) {
        tmem_ld32(sbuf + wg * 64, sv);
        tmem_ld32(sbuf + wg * 64 + 32, sv + 32);
      }
      const int blk = col - (col / p.nb) * p.nb;
      const bool valid = e != 0xFFFFFFFFu;
      int lim = 127;
      // partial row: entry (start + token) of the column-sorted list, head
      const long long prow = (static_cast<long long>(cs.y) + tok) * p.r + head;
      if (valid) {
        const int pos = p.q_off + static_cast<int>(e >> 6);
        if ((pos >> 7) == blk) lim = pos & 127;
      }
      if (ok) tc_wait_ld();
      // Only rows of the local block need the causal mask; the branch is
      // uniform over the warp in the common case.
      const bool full = __all_sync(0xffffffffu, lim == 127);
      if (!full) {
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] = wg * 64 + x <= lim ? sv[x] : -INFINITY;
      }
      // half-row max with three-input max: eight chains of eight values
      float m8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) m8[x] = fmax3(sv[x], sv[x + 8], sv[x + 16]);
#pragma unroll
      for (int b = 24; b < 56; b += 16)
#pragma unroll
        for (int x = 0; x < 8; ++x) m8[x] = fmax3(m8[x], sv[b + x], sv[b + 8 + x]);
#pragma unroll
      for (int x = 0; x < 8; ++x) m8[x] = fmaxf(m8[x], sv[56 + x]);
      const float mloc = fmaxf(fmax3(m8[0], m8[1], m8[2]),
                               fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
      xmax[(par * 2 + wg) * 128 + row] = mloc;
      if (named_bar_or(2, 256, !ok)) break;
      const float mx = fmaxf(mloc, xmax[(par * 2 + (wg ^ 1)) * 128 + row]);
      const float mxs = mx * p.scale_log2;
      // P = 2^(s*scale - max) as bf16, written over the S columns (keys
      // 64 wg .. 64 wg + 63 are packed columns 32 wg .. 32 wg + 31); the sum
      // is of the rounded values the PV product uses, so that the partial
      // output is an exact convex combination of V rows before its own
      // rounding.  Scale-and-shift and the sums run on packed fp32 pairs.
      const uint64_t nm2 = f2_pack(-mxs, -mxs);
      uint64_t l4[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) l4[x] = 0ull;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 a = f2_unpack(ffma2(f2_pack(sv[c * 32 + x], sv[c * 32 + x + 1]), sc2, nm2));
          const float e0 = fast_exp2(a.x);
          const float e1 = fast_exp2(a.y);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
          const uint32_t w = *reinterpret_cast<uint32_t*>(&h2);
          pk[x >> 1] = w;
          // the pair widened exactly (bf16 is the top half of an fp32)
          l4[(x >> 1) & 3] = fadd2(l4[(x >> 1) & 3],
                                   f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
        }
        tmem_st16(sbuf + wg * 32 + c * 16, pk);
      }
      const float2 la = f2_unpack(fadd2(fadd2(l4[0], l4[1]), fadd2(l4[2], l4[3])));
      const float lpart = la.x + la.y;
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&pfull[sb]);
      if (valid && wg == 0) p.w.part_ml[2 * prow] = mxs;
      // the partial sum for the epilogue of this tile
      if (mbar_wait(&lempty[par], ((i >> 1) & 1) ^ 1, abort_flag, p.err)) {
        xsum[(par * 2 + wg) * 128 + row] = lpart;
        mbar_arrive(&lfull[par]);
      } else {
        failed = true;
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    // O row (scaled by 1/l, bf16) -> swizzled staging tile -> TMA stores, one
    // 64-column half of the rows at a time.  Partials are stored in entry
    // order, so the 128 rows of a full tile are one contiguous block: one
    // store per half.  The last, partial tile of a column stores its tokens'
    // r rows one token at a time.  l is the sum of the two softmax
    // warpgroups' partial sums.
    regs_dec<96>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tok = row / p.r, head = row % p.r;
    uint8_t* stage = smem + L::kOffStage;
    uint8_t* srow = stage + row * 128;
    bool stored = false;   // this thread has bulk stores in flight
    int4 td_next = n > 0 ? p.w.tiles[t_begin] : make_int4(0, 0, 0, 0);   // one tile ahead
    for (long long i = 0; i < n; ++i) {
      const int4 td = td_next;   // column, entry start, entries
      if (i + 1 < n) td_next = p.w.tiles[t_begin + i + 1];
      const int ob = static_cast<int>(i % kNO);
      const int par = static_cast<int>(i & 1);
      const bool ok = mbar_wait(&ofull[ob], (i / kNO) & 1, abort_flag, p.err) &&
                      mbar_wait(&lfull[par], (i >> 1) & 1, abort_flag, p.err);
      // the staging tile must be free: own stores read out, then everyone's;
      // and the four warps leave together if a wait gave up
      if (stored) {
        bulk_wait_read0();
        stored = false;
      }
      if (named_bar_or(1, 128, !ok)) break;
      tc_fence_after();
      const float l = xsum[(par * 2) * 128 + row] + xsum[(par * 2 + 1) * 128 + row];
      mbar_arrive(&lempty[par]);
      if (tok < td.z) p.w.part_ml[2 * ((static_cast<long long>(td.y) + tok) * p.r + head) + 1] = l;
      const float il = 1.f / l;
      const uint64_t il2 = f2_pack(il, il);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        if (h > 0) {
          // the staging tile must be free: own stores read out, then everyone's
          if (stored) {
            bulk_wait_read0();
            stored = false;
          }
          named_bar_sync(1, 128);
        }
        float ov[64];
        tmem_ld32(tO + ob * D + lane_off + h * 64, ov);
        tmem_ld32(tO + ob * D + lane_off + h * 64 + 32, ov + 32);
        tc_wait_ld();
        if (h + 1 == D / 64) {
          tc_fence_before();
          mbar_arrive(&ofree[ob]);
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          // scale by 1/l on packed pairs, then round to bf16
          float2 q[4];
#pragma unroll
          for (int y = 0; y < 4; ++y)
            q[y] = f2_unpack(fmul2(f2_pack(ov[8 * x + 2 * y], ov[8 * x + 2 * y + 1]), il2));
          __nv_bfloat162 h0 = __floats2bfloat162_rn(q[0].x, q[0].y);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(q[1].x, q[1].y);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(q[2].x, q[2].y);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(q[3].x, q[3].y);
          uint4* dst = reinterpret_cast<uint4*>(srow + ((x ^ (row & 7)) << 4));
          *dst = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                            *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (td.z == tpt) {
          if (row == 0) {
            tma_store_2d(&tm_ot, stage, h * 64, td.y * p.r);
            bulk_commit_group();
            stored = true;
          }
        } else if (head == 0 && tok < td.z) {
          tma_store_2d(&tm_o, stage + tok * p.r * 128, h * 64, (td.y + tok) * p.r);
          bulk_commit_group();
          stored = true;
        }
      }
    }
    if (stored) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------- 4. combine
// One CTA per (sequence, token): merge the k partials of each of the H heads.
// Partial s of a row holds the normalised output O_s (bf16), its running max
// m_s and sum l_s = sum_j 2^(x_j - m_s) (x in log2 units).  With M = max_s m_s
// and w_s = 2^(m_s - M) l_s:  o = sum_s w_s O_s / sum_s w_s.  The partial of
// (group g, slot s) sits at entry inv[t, g, s] of the column-sorted list.
//
// KL (index-alignment diagnostic, MiniMax Sparse Attention pages, "KL Loss
// Alignment"): w_s / sum_s w_s is the attention mass head h puts on selected
// block s, so the same (m, l) pairs also give, per group g,
//   P_main(s)  = mean over the group's heads of w_s / sum w
//   P_index(s) = softmax over the selected slots of pooled[t, g, sel[s]]
//   kl[t, g]   = sum_s P_main(s) (log P_main(s) - log P_index(s)).
// Eight CTAs per SM (<= 32 registers, no spills): the kernel waits on
// scattered partial reads, so resident warps decide its speed (six CTAs at
// 40 registers ran 13% slower).
template <int D, bool KL>
__global__ void __launch_bounds__(256, 8) combine_kernel(const int32_t* __restrict__ sel,
                                                      const PrefillWs w, uint16_t* __restrict__ o,
                                                      float* __restrict__ lse, int H, int G,
                                                      int r, int k, int T, int q_off,
                                                      const float* __restrict__ pooled,
                                                      float* __restrict__ kl, int nb) {
  constexpr int CH = D / 8;                  // 16-byte chunks per head row
  extern __shared__ float2 sm_ml[];          // [k][H] (m, l), m = -inf for unused slots
  float2* sm_hd = sm_ml + k * H;             // KL only: [H] (M, 1 / den)
  float* sm_z = reinterpret_cast<float*>(sm_hd + (KL ? H : 0));   // KL only: [G][k] pooled
  uint32_t* sm_pos = reinterpret_cast<uint32_t*>(sm_z + (KL ? G * k : 0));   // [G][k] entries
  const long long bt = blockIdx.x;           // b*T + t
  const float2* ml_all = reinterpret_cast<const float2*>(w.part_ml);
  const int32_t* srow = sel + bt * G * k;
  const uint32_t* irow = w.inv + bt * G * k;
  const int lb = (q_off + static_cast<int>(bt % T)) >> 7;   // the query's block
  for (int x = threadIdx.x; x < G * k; x += blockDim.x) {
    const int j = srow[x];
    const bool used = j >= 0 && j <= lb;     // the slots the inversion kept
    sm_pos[x] = used ? irow[x] : 0xFFFFFFFFu;
    if constexpr (KL) sm_z[x] = used ? pooled[(bt * G + x / k) * nb + j] : -INFINITY;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < k * H; x += blockDim.x) {
    const int s = x / H, h = x % H, g = h / r;
    const uint32_t pos = sm_pos[g * k + s];
    sm_ml[x] = pos != 0xFFFFFFFFu ? ml_all[static_cast<long long>(pos) * r + (h - g * r)]
                                  : make_float2(-INFINITY, 0.f);
  }
  __syncthreads();
  for (int item = threadIdx.x; item < H * CH; item += blockDim.x) {
    const int h = item / CH, c = item % CH;
    const int g = h / r, hh = h - g * r;
    float M = -INFINITY;
    for (int s = 0; s < k; ++s) M = fmaxf(M, sm_ml[s * H + h].x);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float den = 0.f;
#pragma unroll 4
    for (int s = 0; s < k; ++s) {
      const float2 ml = sm_ml[s * H + h];
      if (ml.x == -INFINITY) continue;
      const float ws = exp2f(ml.x - M) * ml.y;
      den += ws;
      const long long prow = static_cast<long long>(sm_pos[g * k + s]) * r + hh;
      const uint4 u = __ldcs(reinterpret_cast<const uint4*>(w.part_o + prow * D) + c);
      const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wds[e]));
        acc[2 * e] += ws * f.x;
        acc[2 * e + 1] += ws * f.y;
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;   // no block at all: o = 0, lse = -inf
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 x = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      out[e] = *reinterpret_cast<uint32_t*>(&x);
    }
    *(reinterpret_cast<uint4*>(o + (bt * H + h) * D) + c) = make_uint4(out[0], out[1], out[2], out[3]);
    if (lse && c == 0) lse[bt * H + h] = (M + log2f(den)) / kLog2e;
    if constexpr (KL) {
      if (c == 0) sm_hd[h] = make_float2(M, inv);
    }
  }
  if constexpr (KL) {
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int g = threadIdx.x >> 5; g < G; g += blockDim.x >> 5) {
      const float* zg = sm_z + g * k;
      float zmax = -INFINITY;
      for (int s = lane; s < k; s += 32) zmax = fmaxf(zmax, zg[s]);
      for (int off = 16; off; off >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(~0u, zmax, off));
      float zsum = 0.f;
      for (int s = lane; s < k; s += 32)
        if (zg[s] != -INFINITY) zsum += expf(zg[s] - zmax);
      for (int off = 16; off; off >>= 1) zsum += __shfl_xor_sync(~0u, zsum, off);
      const float log_z = logf(zsum);        // ln P_index(s) = z_s - zmax - log_z
      float acc = 0.f;
      for (int s = lane; s < k; s += 32) {
        if (zg[s] == -INFINITY) continue;
        float pm = 0.f;
        for (int hh = 0; hh < r; ++hh) {
          const int h = g * r + hh;
          const float2 ml = sm_ml[s * H + h];
          const float2 hd = sm_hd[h];
          if (ml.x != -INFINITY) pm += exp2f(ml.x - hd.x) * ml.y * hd.y;
        }
        pm /= static_cast<float>(r);
        if (pm > 0.f) acc += pm * (logf(pm) - (zg[s] - zmax - log_z));
      }
      for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(~0u, acc, off);
      if (lane == 0) kl[bt * G + g] = acc;
    }
  }
}

// One CTA per SM, at most kMaxAttnGrid (the size of the dealing tables).
int attn_grid(const DevCtx* ctx) { return std::min(std::max(ctx->num_sms, 1), kMaxAttnGrid); }

template <int D>
cudaError_t launch_attn(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const AttnParams& p, const DevCtx* ctx,
                        cudaStream_t st) {
  CUtensorMap tq, tk, tv, to, tot;
  const uint64_t rows = static_cast<uint64_t>(s.batch) * s.seq_q * s.n_q_heads;
  const uint64_t dq[2] = {static_cast<uint64_t>(D), rows};
  // [half of the row (stride 128 B)][row (stride 256 B)][64 columns]
  const uint64_t dq3[3] = {64, rows, 2};
  const uint64_t sq3[2] = {static_cast<uint64_t>(D) * 2, 128};
  const uint32_t bq3[3] = {64, 8, 2};
  const uint64_t sq[1] = {static_cast<uint64_t>(D) * 2};
  const uint32_t bq[2] = {64, static_cast<uint32_t>(p.r)};
  // K/V: [B*G][N][d] contiguous, or [P*G][128][d] in pages of one block
  const uint64_t kv_rows = p.pages ? 128 : static_cast<uint64_t>(s.seq_kv);
  const uint64_t kv_mats = p.pages ? static_cast<uint64_t>(p.num_pages) * s.n_kv_heads
                                   : static_cast<uint64_t>(s.batch) * s.n_kv_heads;
  const uint64_t dk[3] = {static_cast<uint64_t>(D), kv_rows, kv_mats};
  const uint64_t sk[2] = {static_cast<uint64_t>(D) * 2, kv_rows * D * 2};
  const uint32_t bk[3] = {64, 128, 1};
  // partial rows: (entry, head) with entries in column order
  const uint64_t prow = static_cast<uint64_t>(s.batch) * s.seq_q * s.topk * s.n_q_heads;
  const uint64_t dpo[2] = {static_cast<uint64_t>(D), prow};
  const uint32_t bpt[2] = {64, 128};
  const bool qmap = p.q3d ? encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dq3, sq3,
                                        bq3, CU_TENSOR_MAP_SWIZZLE_128B)
                           : encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dq, sq, bq,
                                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (!qmap ||
      !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.w.part_o, dpo, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tot, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.w.part_o, dpo, sq, bpt,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = AttnSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kvouter_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    ProfScope ps_("kvouter_attn", st);
    kvouter_attn_kernel<D><<<attn_grid(ctx), kAttnThreads, smem, st>>>(tq, tk, tv, to, tot, p);
  }
  return cudaGetLastError();
}

}  // namespace

size_t prefill_workspace_bytes(const msa_shape& s) { return carve_bytes(s); }

constexpr size_t kHistSmemMax = 200u * 1024u;
constexpr size_t kCombineSmemMax = 227u * 1024u;    // the opt-in maximum per CTA
constexpr size_t kDefaultSmem = 48u * 1024u;

static size_t combine_smem_bytes(const msa_shape& s, bool with_kl) {
  const size_t H = s.n_q_heads, G = s.n_kv_heads, k = s.topk;
  return 8 * k * H + (with_kl ? 8 * H + 4 * G * k : 0) + 4 * G * k;
}

bool prefill_shape_supported(const msa_shape& s) {
  const size_t nb = static_cast<size_t>(ceil_div(s.seq_kv, 128));
  const PrefillWs w = carve(s, nullptr);
  const long long nent = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads * s.topk;
  // 32-bit columns, tile ids and entry positions
  return 8 * nb <= kHistSmemMax && combine_smem_bytes(s, true) <= kCombineSmemMax &&
         w.ncol < (1ll << 31) && w.max_tiles < (1ll << 31) && nent < (1ll << 32);
}

cudaError_t launch_sparse_prefill(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const int32_t* sel, uint16_t* o,
                                  float* lse, void* ws, cudaStream_t st, const float* pooled,
                                  float* kl, PageTable pages) {
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
  if (!prefill_shape_supported(s)) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(sel_invert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(hsmem));
  if (e != cudaSuccess) return e;
  {
    ProfScope ps_("sel_count", st);
    sel_invert_kernel<<<hgrid, 256, hsmem, st>>>(sel, w, s.seq_q, s.n_kv_heads, s.topk, nb,
                                                 s.q_offset, 0, ctx->err);
  }
  {
    ProfScope ps_("scan_columns", st);
    scan_columns_kernel<<<1, 1024, 0, st>>>(w, tpt);
  }
  {
    ProfScope ps_("sel_scatter", st);
    sel_invert_kernel<<<hgrid, 256, hsmem, st>>>(sel, w, s.seq_q, s.n_kv_heads, s.topk, nb,
                                                 s.q_offset, 1, ctx->err);
  }
  // chunk rotation between consecutive segments: spreads the segments'
  // last chunks over the grid
  const int grid = attn_grid(ctx);
  const int rot = static_cast<int>(std::max<long long>(1, grid / std::max<long long>(1, std::min<long long>(w.nseg, grid))));
  {
    ProfScope ps_("plan_ctas", st);
    plan_ctas_kernel<<<1, 1024, 0, st>>>(w, nb, grid, rot);
  }
  {
    ProfScope ps_("make_tiles", st);
    make_tiles_kernel<<<static_cast<unsigned>(ceil_div(w.max_tiles, 256)), 256, 0, st>>>(
        w, tpt, nb, grid, rot);
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
  p.q3d = (r == 8 && s.head_dim == 128) ? 1 : 0;
  p.pages = pages.table;
  p.num_pages = pages.num_pages;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(s.head_dim));
  e = s.head_dim == 128 ? launch_attn<128>(s, q, k, v, p, ctx, st)
                        : launch_attn<64>(s, q, k, v, p, ctx, st);
  if (e != cudaSuccess) return e;
  const unsigned ntok = static_cast<unsigned>(static_cast<long long>(s.batch) * s.seq_q);
  const bool with_kl = kl != nullptr;
  const size_t csmem = combine_smem_bytes(s, with_kl);
  if (csmem > kDefaultSmem) {
    // many heads x many slots: opt in to more than the default 48 KB
    const void* fn = s.head_dim == 128
                         ? (with_kl ? reinterpret_cast<const void*>(combine_kernel<128, true>)
                                    : reinterpret_cast<const void*>(combine_kernel<128, false>))
                         : (with_kl ? reinterpret_cast<const void*>(combine_kernel<64, true>)
                                    : reinterpret_cast<const void*>(combine_kernel<64, false>));
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(csmem));
    if (e != cudaSuccess) return e;
  }
  {
    ProfScope ps_(with_kl ? "combine_kl" : "combine", st);
    const int H = s.n_q_heads, G = s.n_kv_heads, kk = s.topk, T = s.seq_q, qo = s.q_offset;
    if (s.head_dim == 128 && with_kl)
      combine_kernel<128, true><<<ntok, 256, csmem, st>>>(sel, w, o, lse, H, G, r, kk, T, qo,
                                                          pooled, kl, nb);
    else if (s.head_dim == 128)
      combine_kernel<128, false><<<ntok, 256, csmem, st>>>(sel, w, o, lse, H, G, r, kk, T, qo,
                                                           nullptr, nullptr, nb);
    else if (with_kl)
      combine_kernel<64, true><<<ntok, 256, csmem, st>>>(sel, w, o, lse, H, G, r, kk, T, qo,
                                                         pooled, kl, nb);
    else
      combine_kernel<64, false><<<ntok, 256, csmem, st>>>(sel, w, o, lse, H, G, r, kk, T, qo,
                                                          nullptr, nullptr, nb);
  }
  return cudaGetLastError();
}

}  // namespace msa

namespace msa {
cudaError_t set_wait_limit_prefill(uint64_t ns) { return set_wait_limit_here(ns); }
}  // namespace msa
