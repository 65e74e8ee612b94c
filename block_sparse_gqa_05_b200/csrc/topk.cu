// Block top-k with the local block forced in (yhxrc.cn article, section 第一步
// "TopK"; lumi-systems AI news: per-group independent, exponential-free top-k;
// lefilia.fr: the local block is always included, 16 blocks of 128 tokens).
//
// One warp per (sequence, token, group) row, or one CTA per row when there
// are few long rows (decode).  Candidates are blocks 0..b_t-1;
// the order is (pooled score descending, block index ascending), encoded as a
// 64-bit key ((order-preserving score bits) << 32 | ~index) so every compare
// is exact and ties resolve to the lower block index.  Each chunk of 512
// scores (16 per lane) is filtered against a threshold that provably keeps the (k-1) best
// (the (k-1)-th largest of the 32 per-lane maxima, or the running (k-1)-th
// best), and the survivors are merged into the running list with a warp
// bitonic sort.  No exponentials, no full sort of the row.  Thresholds are
// compared on the 32-bit score keys; only the survivors get 64-bit keys.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;
constexpr int kPer = 16;             // scores per lane per chunk
constexpr int kChunk = 32 * kPer;    // scores per warp per chunk
constexpr int kScratch = 128;        // per-warp merge buffer (64-bit keys)

MSA_DEV uint64_t shfl_xor64(uint64_t x, int m) {
  uint32_t lo = static_cast<uint32_t>(x), hi = static_cast<uint32_t>(x >> 32);
  lo = __shfl_xor_sync(0xffffffffu, lo, m);
  hi = __shfl_xor_sync(0xffffffffu, hi, m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

MSA_DEV uint64_t shfl64(uint64_t x, int src) {
  uint32_t lo = static_cast<uint32_t>(x), hi = static_cast<uint32_t>(x >> 32);
  lo = __shfl_sync(0xffffffffu, lo, src);
  hi = __shfl_sync(0xffffffffu, hi, src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Composite key: larger = better; ties in score resolved by the lower index.
MSA_DEV uint64_t make_key(uint32_t ord_score, int idx) {
  return (static_cast<uint64_t>(ord_score) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}
MSA_DEV int key_index(uint64_t key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

// Descending bitonic sort of 32*S 64-bit keys; element e = s*32 + lane in x[s].
template <int S>
MSA_DEV void warp_sort_desc(uint64_t (&x)[S]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32 * S; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const int ps = s ^ (j >> 5);
          if (ps > s) {
            const bool desc = ((s * 32 + lane) & k) == 0;
            const uint64_t a = x[s], b = x[ps];
            const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
            x[s] = desc ? hi : lo;
            x[ps] = desc ? lo : hi;
          }
        }
      } else {
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const uint64_t y = shfl_xor64(x[s], j);
          const bool desc = ((s * 32 + lane) & k) == 0;
          const bool take_max = desc == ((lane & j) == 0);
          const uint64_t mx = x[s] > y ? x[s] : y, mn = x[s] > y ? y : x[s];
          x[s] = take_max ? mx : mn;
        }
      }
    }
  }
}

// Descending bitonic sort of 32 32-bit values, one per lane.
MSA_DEV uint32_t warp_sort_desc32(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
      const bool take_max = ((lane & k) == 0) == ((lane & j) == 0);
      x = take_max ? max(x, y) : min(x, y);
    }
  }
  return x;
}

// Sorts the first m (<= 32*S) keys of buf descending into best (elements
// lane and 32+lane); slots past m count as empty (key 0).
template <int S>
__device__ __noinline__ void sort_buffer(const uint64_t* buf, int m, uint64_t& best0,
                                         uint64_t& best1) {
  const int lane = threadIdx.x & 31;
  uint64_t x[S];
#pragma unroll
  for (int s = 0; s < S; ++s) x[s] = s * 32 + lane < m ? buf[s * 32 + lane] : 0ull;
  warp_sort_desc<S>(x);
  best0 = x[0];
  best1 = S > 1 ? x[1 % S] : 0ull;
}

// The 64 largest of two descending lists of 64 keys (elements lane and
// 32 + lane of a and of b), descending: pairing a[i] with b[63-i] leaves the
// 64 largest as one bitonic sequence, which six half-cleaner stages sort.
MSA_DEV void merge_top64(uint64_t& a0, uint64_t& a1, uint64_t b0, uint64_t b1) {
  const int lane = threadIdx.x & 31;
  const uint64_t r0 = shfl64(b1, 31 - lane), r1 = shfl64(b0, 31 - lane);
  uint64_t c0 = a0 > r0 ? a0 : r0, c1 = a1 > r1 ? a1 : r1;
  const uint64_t hi = c0 > c1 ? c0 : c1, lo = c0 > c1 ? c1 : c0;
  c0 = hi;
  c1 = lo;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const bool take_max = (lane & j) == 0;
    const uint64_t y0 = shfl_xor64(c0, j), y1 = shfl_xor64(c1, j);
    c0 = take_max ? (c0 > y0 ? c0 : y0) : (c0 > y0 ? y0 : c0);
    c1 = take_max ? (c1 > y1 ? c1 : y1) : (c1 > y1 ? y1 : c1);
  }
  a0 = c0;
  a1 = c1;
}

// best0/best1: running list (elements lane, 32+lane, descending); nk: one new
// key per lane (0 = none).  Keeps the 64 largest of the 96.
__device__ __noinline__ void merge128(uint64_t& best0, uint64_t& best1, uint64_t nk) {
  uint64_t xk[4] = {best0, best1, nk, 0ull};
  warp_sort_desc<4>(xk);
  best0 = xk[0];
  best1 = xk[1];
}

// Scans chunks c0, c0 + cs, c0 + 2 cs, ... (kChunk candidates each, in
// increasing order) of one row's n candidates into the running list ``best``
// (descending; elements lane and 32 + lane; ``have`` valid, at most kk).
MSA_DEV void scan_chunks(const float* __restrict__ src, int n, int kk, bool vec, int c0, int cs,
                         uint64_t* buf, uint64_t (&best)[2], int& have) {
  const int lane = threadIdx.x & 31;
  for (int base = c0 * kChunk; base < n; base += cs * kChunk) {
    // one warp per row: two chunks ahead toward L2 (16 lanes, a 128-byte
    // line each), so that a long row's loads do not wait on DRAM
    if (cs == 1) {
      const int ahead = base + 2 * kChunk + lane * 32;
      if (lane < kChunk / 32 && ahead < n) prefetch_l2(src + ahead);
    }
    // this lane's scores: block base + x*128 + lane*4 + e, as order-preserving keys
    uint32_t uk[kPer];
#pragma unroll
    for (int x = 0; x < kPer / 4; ++x) {
      const int i0 = base + x * 128 + lane * 4;
      float4 f;
      if (vec && i0 + 3 < n) {
        f = __ldg(reinterpret_cast<const float4*>(src + i0));
      } else {
        f.x = i0 < n ? __ldg(src + i0) : 0.f;
        f.y = i0 + 1 < n ? __ldg(src + i0 + 1) : 0.f;
        f.z = i0 + 2 < n ? __ldg(src + i0 + 2) : 0.f;
        f.w = i0 + 3 < n ? __ldg(src + i0 + 3) : 0.f;
      }
      uk[4 * x] = i0 < n ? float_order_key(f.x) : 0u;
      uk[4 * x + 1] = i0 + 1 < n ? float_order_key(f.y) : 0u;
      uk[4 * x + 2] = i0 + 2 < n ? float_order_key(f.z) : 0u;
      uk[4 * x + 3] = i0 + 3 < n ? float_order_key(f.w) : 0u;
    }
    // score threshold that keeps every member of the new top-kk
    uint32_t tau;
    if (have >= kk) {
      // every later block has a larger index than the list's members, so a
      // score equal to the current kk-th best can no longer enter: strict >
      const uint32_t kth = static_cast<uint32_t>(shfl64(best[(kk - 1) >> 5], (kk - 1) & 31) >> 32);
      if (kth == 0xFFFFFFFFu) continue;
      tau = kth + 1u;
    } else if (kk <= 32) {
      uint32_t lmax = 0u;
#pragma unroll
      for (int x = 0; x < kPer; ++x) lmax = max(lmax, uk[x]);
      tau = __shfl_sync(0xffffffffu, warp_sort_desc32(lmax), kk - 1);
    } else {
      tau = 0u;
    }
    tau = max(tau, 1u);
    int cnt = 0;
#pragma unroll
    for (int x = 0; x < kPer; ++x) cnt += uk[x] >= tau ? 1 : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total == 0) continue;
    const int keep = have < kk ? have : kk;
    const int m = keep + total;
    if (m <= kScratch) {
      // running list and survivors into the warp buffer, one sort of <= 128
      if (lane < keep) buf[lane] = best[0];
      if (lane + 32 < keep) buf[32 + lane] = best[1];
      int slot = keep + incl - cnt;
#pragma unroll
      for (int x = 0; x < kPer; ++x) {
        if (uk[x] >= tau) {
          const int i = base + (x >> 2) * 128 + lane * 4 + (x & 3);
          buf[slot++] = make_key(uk[x], i);
        }
      }
      __syncwarp();
      if (m <= 32) {
        uint64_t x1[1];
        x1[0] = lane < m ? buf[lane] : 0ull;
        warp_sort_desc<1>(x1);
        best[0] = x1[0];
        best[1] = 0ull;
      } else if (m <= 64) {
        sort_buffer<2>(buf, m, best[0], best[1]);
      } else {
        sort_buffer<4>(buf, m, best[0], best[1]);
      }
      __syncwarp();
    } else {
      // rare: merge the survivors one register slot at a time
#pragma unroll
      for (int x = 0; x < kPer; ++x) {
        const bool take = uk[x] >= tau;
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        if (bal != 0u) {
          const int i = base + (x >> 2) * 128 + lane * 4 + (x & 3);
          merge128(best[0], best[1], take ? make_key(uk[x], i) : 0ull);
        }
      }
    }
    have = min(m, kk);
    if (lane >= kk) best[0] = 0ull;
    if (lane + 32 >= kk) best[1] = 0ull;
  }
}

// Writes a row's selection: the kk chosen blocks (best, descending) plus the
// local block bt, ascending, then -1 padding up to k.
MSA_DEV void write_selection(int32_t* out, const uint64_t (&best)[2], int kk, int bt, int k) {
  const int lane = threadIdx.x & 31;
  if (kk < 32) {
    const uint32_t idx = lane < kk ? static_cast<uint32_t>(key_index(best[0]))
                                   : (lane == kk ? static_cast<uint32_t>(bt) : 0xFFFFFFFFu);
    const uint32_t sorted = ~warp_sort_desc32(~idx);   // ascending
    if (lane < k) out[lane] = lane <= kk ? static_cast<int32_t>(sorted) : -1;
    for (int i = lane + 32; i < k; i += 32) out[i] = -1;
  } else {
    const uint32_t i0 = static_cast<uint32_t>(key_index(best[0]));
    const int e1 = lane + 32;
    const uint32_t i1 = e1 < kk ? static_cast<uint32_t>(key_index(best[1]))
                                : (e1 == kk ? static_cast<uint32_t>(bt) : 0xFFFFFFFFu);
    uint64_t xk[2] = {static_cast<uint64_t>(~i0), static_cast<uint64_t>(~i1)};
    warp_sort_desc<2>(xk);
    const uint32_t s0 = ~static_cast<uint32_t>(xk[0]), s1 = ~static_cast<uint32_t>(xk[1]);
    if (lane < k) out[lane] = lane <= kk ? static_cast<int32_t>(s0) : -1;
    if (e1 < k) out[e1] = e1 <= kk ? static_cast<int32_t>(s1) : -1;
  }
}

// Rows whose selection needs no ranking: every causal block fits (kk == n)
// or only the local block is asked for (kk == 0).  Returns true if handled.
MSA_DEV bool write_trivial(int32_t* out, int n, int kk, int bt, int k) {
  const int lane = threadIdx.x & 31;
  if (kk == n) {
    for (int i = lane; i < k; i += 32) out[i] = i <= bt ? i : -1;
    return true;
  }
  if (kk == 0) {
    for (int i = lane; i < k; i += 32) out[i] = i == 0 ? bt : -1;
    return true;
  }
  return false;
}

// One warp per row: for many rows (prefill).  Five CTAs per SM (48
// registers): the kernel waits on its loads, so resident warps matter more
// than the few registers it spills.
__global__ void __launch_bounds__(kWarps * 32, 5)
    block_topk_kernel(const float* __restrict__ pooled, int32_t* __restrict__ sel,
                      long long rows, int T, int G, int q_off, int nb, int k,
                      const int32_t* __restrict__ lens, int N, uint32_t* err) {
  __shared__ uint64_t scratch[kWarps][kScratch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* buf = scratch[warp];
  const long long nwarps = static_cast<long long>(gridDim.x) * kWarps;
  griddep_launch_dependents();   // the attention may launch (it waits for this kernel)
  griddep_wait();                // the pooled scores of the kernel before
  const bool vec = (nb & 3) == 0;
  // query position of row rr (rows < 2^31, checked by the API: 32-bit index math)
  auto row_pos = [&](long long rr) {
    const uint32_t tg = static_cast<uint32_t>(rr) / static_cast<uint32_t>(G);
    const int t = static_cast<int>(tg % static_cast<uint32_t>(T));
    return lens ? ragged_len(lens, static_cast<int>(tg / static_cast<uint32_t>(T)), N, err) - 1
                : q_off + t;
  };
  for (long long r = static_cast<long long>(blockIdx.x) * kWarps + warp; r < rows; r += nwarps) {
    // the warp's next row: its first two chunks of candidate scores toward
    // L2 (one 128-byte line per lane) while this row is ranked, so that its
    // first loads do not wait on DRAM
    if (r + nwarps < rows) {
      const float* nsrc = pooled + (r + nwarps) * nb;
      const int nn = min(row_pos(r + nwarps) >> 7, 2 * kChunk);
      if (lane * 32 < nn) prefetch_l2(nsrc + lane * 32);
    }
    const int pos = row_pos(r);
    const int bt = pos >> 7;
    const int n = bt;                         // candidates 0 .. bt-1
    const int kk = min(k - 1, n);
    int32_t* out = sel + r * k;
    if (write_trivial(out, n, kk, bt, k)) continue;
    uint64_t best[2] = {0ull, 0ull};
    int have = 0;
    scan_chunks(pooled + r * nb, n, kk, vec, 0, 1, buf, best, have);
    write_selection(out, best, kk, bt, k);
  }
}

// One CTA per row: for few long rows (decode).  Warp w scans chunks w,
// w + kWarps, ...; the kWarps lists are then merged pairwise in a tree (each
// merge keeps the 64 best of two sorted lists of at most 63).
__global__ void __launch_bounds__(kWarps * 32)
    block_topk_row_cta_kernel(const float* __restrict__ pooled, int32_t* __restrict__ sel,
                              int T, int G, int q_off, int nb, int k,
                              const int32_t* __restrict__ lens, int N, uint32_t* err) {
  __shared__ uint64_t scratch[kWarps][kScratch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = blockIdx.x;
  griddep_launch_dependents();   // the attention may launch (it waits for this kernel)
  griddep_wait();                // the pooled scores of the kernel before
  const uint32_t tg = static_cast<uint32_t>(r) / static_cast<uint32_t>(G);
  const int t = static_cast<int>(tg % static_cast<uint32_t>(T));
  const int pos = lens ? ragged_len(lens, static_cast<int>(tg / static_cast<uint32_t>(T)), N, err) - 1
                       : q_off + t;
  const int bt = pos >> 7;
  const int n = bt;
  const int kk = min(k - 1, n);
  int32_t* out = sel + r * k;
  if (kk == n || kk == 0) {
    if (warp == 0) write_trivial(out, n, kk, bt, k);
    return;
  }
  uint64_t best[2] = {0ull, 0ull};
  int have = 0;
  scan_chunks(pooled + r * nb, n, kk, (nb & 3) == 0, warp, kWarps, scratch[warp], best, have);
  __syncwarp();
  scratch[warp][lane] = best[0];
  scratch[warp][32 + lane] = best[1];
  __syncthreads();
#pragma unroll
  for (int span = 1; span < kWarps; span <<= 1) {
    if ((warp & (2 * span - 1)) == 0) {
      uint64_t a0 = scratch[warp][lane], a1 = scratch[warp][32 + lane];
      merge_top64(a0, a1, scratch[warp + span][lane], scratch[warp + span][32 + lane]);
      __syncwarp();
      scratch[warp][lane] = a0;
      scratch[warp][32 + lane] = a1;
    }
    __syncthreads();
  }
  if (warp == 0) {
    best[0] = lane < kk ? scratch[0][lane] : 0ull;
    best[1] = lane + 32 < kk ? scratch[0][32 + lane] : 0ull;
    write_selection(out, best, kk, bt, k);
  }
}

}  // namespace

cudaError_t launch_block_topk(const msa_shape& s, const float* pooled, int32_t* sel,
                              cudaStream_t st, const int32_t* lens) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  const long long rows = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads;
  const int nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  // Few long rows (decode) leave most warps of the one-warp-per-row kernel
  // idle: give each row a CTA instead.
  if (rows <= 4LL * ctx->num_sms && nb > kChunk) {
    ProfScope ps_("block_topk", st);
    // may start while the index scan before it finishes (it waits for it)
    const cudaError_t e = launch_dependent(block_topk_row_cta_kernel,
                                           dim3(static_cast<unsigned>(rows)), dim3(kWarps * 32), 0,
                                           st, pooled, sel, s.seq_q, s.n_kv_heads, s.q_offset, nb,
                                           s.topk, lens, s.seq_kv, ctx->err);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  long long blocks = (rows + kWarps - 1) / kWarps;
  const long long cap = static_cast<long long>(ctx->num_sms) * 32;
  if (blocks > cap) blocks = cap;
  {
    ProfScope ps_("block_topk", st);
    const cudaError_t e = launch_dependent(block_topk_kernel, dim3(static_cast<unsigned>(blocks)),
                                           dim3(kWarps * 32), 0, st, pooled, sel, rows, s.seq_q,
                                           s.n_kv_heads, s.q_offset, nb, s.topk, lens, s.seq_kv,
                                           ctx->err);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace msa
