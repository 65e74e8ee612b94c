// Block top-k with the local block forced in (yhxrc.cn article, section 第一步
// "TopK"; lumi-systems AI news: per-group independent, exponential-free top-k;
// lefilia.fr: the local block is always included, 16 blocks of 128 tokens).
//
// One warp per (sequence, token, group) row.  Candidates are blocks 0..b_t-1;
// the order is (pooled score descending, block index ascending), encoded as a
// 64-bit key ((order-preserving score bits) << 32 | ~index) so every compare
// is exact and ties resolve to the lower block index.  Each chunk of 1024
// scores is filtered against a threshold that provably keeps the (k-1) best
// (the (k-1)-th largest of the 32 per-lane maxima, or the running (k-1)-th
// best), and the survivors are merged into the running list with a warp
// bitonic sort.  No exponentials, no full sort of the row.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;
constexpr int kChunk = 1024;   // scores held per warp at a time (32 per lane)

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

MSA_DEV uint64_t make_key(float score, int idx) {
  return (static_cast<uint64_t>(float_order_key(score)) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}
MSA_DEV int key_index(uint64_t key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

// Descending bitonic sort of 32*S keys; element e = s*32 + lane lives in x[s].
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
          const bool lower = (lane & j) == 0;
          const bool take_max = (desc == lower);
          const uint64_t mx = x[s] > y ? x[s] : y, mn = x[s] > y ? y : x[s];
          x[s] = take_max ? mx : mn;
        }
      }
    }
  }
}

// best0/best1: running list (elements lane, 32+lane, descending); nk: one new
// key per lane (0 = none).  Keeps the 64 largest of the 96.
__device__ __noinline__ void merge128(uint64_t& best0, uint64_t& best1, uint64_t nk) {
  uint64_t xk[4] = {best0, best1, nk, 0ull};
  warp_sort_desc<4>(xk);
  best0 = xk[0];
  best1 = xk[1];
}

__global__ void __launch_bounds__(kWarps * 32)
    block_topk_kernel(const float* __restrict__ pooled, int32_t* __restrict__ sel,
                      long long rows, int T, int G, int q_off, int nb, int k) {
  __shared__ uint64_t scratch[kWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nwarps = static_cast<long long>(gridDim.x) * kWarps;
  const bool vec = (nb & 3) == 0;
  for (long long r = static_cast<long long>(blockIdx.x) * kWarps + warp; r < rows; r += nwarps) {
    const int t = static_cast<int>((r / G) % T);
    const int bt = (q_off + t) >> 7;
    const int n = bt;                         // candidates 0 .. bt-1
    const int kk = min(k - 1, n);
    int32_t* out = sel + r * k;
    if (kk == n) {                            // every causal block fits
      for (int i = lane; i < k; i += 32) out[i] = i <= bt ? i : -1;
      continue;
    }
    if (kk == 0) {
      for (int i = lane; i < k; i += 32) out[i] = i == 0 ? bt : -1;
      continue;
    }
    const float* src = pooled + r * nb;
    uint64_t best[2] = {0ull, 0ull};          // sorted descending: element lane / lane+32
    int have = 0;                             // valid entries in best
    for (int base = 0; base < n; base += kChunk) {
      float v[32];
      if (vec) {
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int i0 = base + x * 128 + lane * 4;
          if (i0 + 3 < n) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(src + i0));
            v[4 * x] = f.x; v[4 * x + 1] = f.y; v[4 * x + 2] = f.z; v[4 * x + 3] = f.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[4 * x + e] = i0 + e < n ? __ldg(src + i0 + e) : 0.f;
          }
        }
      } else {
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = base + x * 128 + lane * 4 + e;
            v[4 * x + e] = i < n ? __ldg(src + i) : 0.f;
          }
      }
      // element (x, e) of this lane has block index base + x*128 + lane*4 + e
      uint64_t lmax = 0ull;
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = base + x * 128 + lane * 4 + e;
          const uint64_t key = i < n ? make_key(v[4 * x + e], i) : 0ull;
          lmax = key > lmax ? key : lmax;
        }
      uint64_t tau = 0ull;
      if (kk <= 32) {
        uint64_t m1[1] = {lmax};
        warp_sort_desc<1>(m1);
        tau = shfl64(m1[0], kk - 1);
      }
      if (have >= kk) {
        const uint64_t run = shfl64(best[(kk - 1) >> 5], (kk - 1) & 31);
        tau = run > tau ? run : tau;
      }
      // count survivors (key >= tau, key > 0)
      int cnt = 0;
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = base + x * 128 + lane * 4 + e;
          const uint64_t key = i < n ? make_key(v[4 * x + e], i) : 0ull;
          cnt += (key != 0ull && key >= tau) ? 1 : 0;
        }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (total == 0) continue;
      const int keep_have = have < kk ? have : kk;
      if (kk <= 32 && keep_have + total <= 32) {
        // fast path: one 32-wide sort of (running list + survivors)
        int slot = incl - cnt;
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = base + x * 128 + lane * 4 + e;
            const uint64_t key = i < n ? make_key(v[4 * x + e], i) : 0ull;
            if (key != 0ull && key >= tau) scratch[warp][slot++] = key;
          }
        __syncwarp();
        uint64_t xk[1];
        xk[0] = lane < keep_have ? best[0]
                                 : (lane - keep_have < total ? scratch[warp][lane - keep_have] : 0ull);
        __syncwarp();
        warp_sort_desc<1>(xk);
        best[0] = xk[0];
        best[1] = 0ull;
        have = keep_have + total;
      } else {
        // general path: merge survivors one register slot at a time into the
        // list with a 128-wide sort (list in elements 0..63, new in 64..95)
#pragma unroll
        for (int x = 0; x < 8; ++x) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = base + x * 128 + lane * 4 + e;
            const uint64_t key = i < n ? make_key(v[4 * x + e], i) : 0ull;
            const bool take = key != 0ull && key >= tau;
            const unsigned bal = __ballot_sync(0xffffffffu, take);
            if (bal != 0u) {
              merge128(best[0], best[1], take ? key : 0ull);
              have += __popc(bal);
            }
          }
        }
        if (kk <= 32) best[1] = 0ull;
      }
      if (have > kk) have = kk;
      // keep only the kk best
      if (lane >= kk) best[0] = 0ull;
      if (lane + 32 >= kk) best[1] = 0ull;
    }
    // output: the kk chosen blocks plus bt, ascending, then -1 padding
    if (kk < 32) {
      uint32_t idx = lane < kk ? static_cast<uint32_t>(key_index(best[0]))
                               : (lane == kk ? static_cast<uint32_t>(bt) : 0xFFFFFFFFu);
      uint64_t xk[1] = {static_cast<uint64_t>(~idx)};   // descending ~idx = ascending idx
      warp_sort_desc<1>(xk);
      const uint32_t sorted = ~static_cast<uint32_t>(xk[0]);
      if (lane < k) out[lane] = lane <= kk ? static_cast<int32_t>(sorted) : -1;
      for (int i = lane + 32; i < k; i += 32) out[i] = -1;
    } else {
      uint32_t i0 = static_cast<uint32_t>(key_index(best[0]));
      const int e1 = lane + 32;
      uint32_t i1 = e1 < kk ? static_cast<uint32_t>(key_index(best[1]))
                            : (e1 == kk ? static_cast<uint32_t>(bt) : 0xFFFFFFFFu);
      uint64_t xk[2] = {static_cast<uint64_t>(~i0), static_cast<uint64_t>(~i1)};
      warp_sort_desc<2>(xk);
      const uint32_t s0 = ~static_cast<uint32_t>(xk[0]), s1 = ~static_cast<uint32_t>(xk[1]);
      if (lane < k) out[lane] = lane <= kk ? static_cast<int32_t>(s0) : -1;
      if (e1 < k) out[e1] = e1 <= kk ? static_cast<int32_t>(s1) : -1;
    }
  }
}

}  // namespace

cudaError_t launch_block_topk(const msa_shape& s, const float* pooled, int32_t* sel,
                              cudaStream_t st) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  const long long rows = static_cast<long long>(s.batch) * s.seq_q * s.n_kv_heads;
  const int nb = static_cast<int>(ceil_div(s.seq_kv, 128));
  long long blocks = (rows + kWarps - 1) / kWarps;
  const long long cap = static_cast<long long>(ctx->num_sms) * 32;
  if (blocks > cap) blocks = cap;
  block_topk_kernel<<<static_cast<unsigned>(blocks), kWarps * 32, 0, st>>>(
      pooled, sel, rows, s.seq_q, s.n_kv_heads, s.q_offset, nb, s.topk);
  return cudaGetLastError();
}

}  // namespace msa
