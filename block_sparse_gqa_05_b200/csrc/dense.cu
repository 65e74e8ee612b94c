// Dense causal GQA prefill: every query attends every key x <= p_t (Notion
// note "Minimax sparse Attention", GQA definition; the baseline the MSA pages
// compare against: hamidun.com "Principais resultados", lumi-systems AI news).
//
// Q-outer flash attention on tcgen05.  One CTA per (sequence, group, tile of
// 128/r tokens): the tile's 128 rows are its tokens x the group's r heads, all
// sharing the group's K/V.  The CTA streams the causal key blocks 0..b_t
// through two TMA stages; per block S = Q K^T lands in TMEM, the softmax
// warpgroup turns it into P (bf16, written over S) with an online maximum, and
// O += P V accumulates in TMEM.  O is rescaled only when a row maximum grows by
// more than 2^8 over the reference it was accumulated with (P stays below 2^8
// otherwise), which waits for the previous PV.  CTAs of one group run side by
// side, so each K/V block is read from HBM about once per wave of CTAs.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 softmax/epilogue
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

struct DenseParams {
  uint16_t* o;
  float* lse;
  uint32_t* err;
  int T, N, H, G, r, q_off, tpt, ntile;   // ntile: query tiles per (sequence, group)
  float scale_log2;
};

template <int D>
struct DenseSmem {
  static constexpr uint32_t kTile = 128u * D * 2u;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kTile;            // 2 stages
  static constexpr uint32_t kOffV = 3 * kTile;        // 2 stages
  static constexpr uint32_t kOffBar = 5 * kTile;
  static constexpr uint32_t kBytes = kOffBar + 256;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dense_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DenseParams p) {
  using L = DenseSmem<D>;
  constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* qfull = bars;          // [1]
  uint64_t* kvfull = bars + 1;     // [2]
  uint64_t* kvempty = bars + 3;    // [2]
  uint64_t* sfull = bars + 5;      // [2]
  uint64_t* pfull = bars + 7;      // [2]
  uint64_t* pvdone = bars + 9;     // [1] one arrival per PV
  uint64_t* mma_drain = bars + 10; // [1] the MMA thread's last commit before exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tiles of one group are consecutive blocks: CTAs resident together share K/V
  const int tile = blockIdx.x % p.ntile;
  const int bg = blockIdx.x / p.ntile;
  const int b = bg / p.G, g = bg % p.G;
  const int t0 = tile * p.tpt;
  const int t_last = min(t0 + p.tpt, p.T) - 1;
  const int nblk = (p.q_off + t_last) / 128 + 1;     // causal key blocks of the tile

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kvfull[i], 1);
      mbar_init(&kvempty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 128);
    }
    mbar_init(pvdone, 1);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (uint32_t x = threadIdx.x; x < L::kTile / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[x] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;          // S/P buffers at [0,128) and [128,256)
  const uint32_t tO = tmem + 256;    // O at [256, 256+D)

  if (warp == 0) {
    // ----------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int ntok = t_last - t0 + 1;
      mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(ntok * p.r * D * 2));
      for (int j = 0; j < ntok; ++j) {
        const int row = (b * p.T + t0 + j) * p.H + g * p.r;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(smem + L::kOffQ + c * 16384 + j * p.r * 128, &tm_q, qfull, c * 64, row);
      }
      int armed = 0;   // K/V blocks whose loads were issued
      for (int j = 0; j < nblk; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kvempty[st], ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&kvfull[st], 2 * L::kTile);
        ++armed;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem + L::kOffK + st * L::kTile + c * 16384, &tm_k, &kvfull[st], c * 64,
                      j * 128, bg);
          tma_load_3d(smem + L::kOffV + st * L::kTile + c * 16384, &tm_v, &kvfull[st], c * 64,
                      j * 128, bg);
        }
      }
      // every load issued lands before the CTA may exit
      mbar_drain(qfull, 0);
      for (int j = armed > 2 ? armed - 2 : 0; j < armed; ++j) mbar_drain(&kvfull[j & 1], (j >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // S(0), S(1), then per block j: PV(j), S(j+2).  MMAs of one thread run in
    // issue order, so S(j+2) may overwrite the S/P buffer of block j after PV(j).
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, abort_flag, p.err);
      const uint32_t qa = smem_u32(smem + L::kOffQ);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&kvfull[st], (j >> 1) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + L::kOffK + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          tc_mma_ss(tS + st * 128, smem_desc(qa + off, 16, 1024, 2),
                    smem_desc(ka + off, 16, 1024, 2), kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&sfull[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nblk > 1) ok = issue_s(1);
      for (int j = 0; ok && j < nblk; ++j) {
        const int st = j & 1;
        if (!(ok = mbar_wait(&pfull[st], (j >> 1) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        const uint32_t va = smem_u32(smem + L::kOffV + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bd = smem_desc(va + ks * 16 * 128, 16384, 1024, 2);
          tc_mma_ts(tO, tS + st * 128 + ks * 8, bd, kIdescO, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(pvdone);
        tc_commit(&kvempty[st]);
        if (j + 2 < nblk && !(ok = issue_s(j + 2))) break;
      }
      // every MMA issued completes before TMEM is released
      tc_drain(mma_drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int tok = row / p.r, head = row % p.r;
    const int t = t0 + tok;
    const bool valid = t <= t_last;
    const int pos = p.q_off + (valid ? t : t_last);
    float m_ref = -INFINITY;   // reference max of the accumulated O (log2 units)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int st = j & 1;
      const uint32_t sbuf = tS + st * 128 + lane_off;
      if (!(ok = mbar_wait(&sfull[st], (j >> 1) & 1, abort_flag, p.err))) break;
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(sbuf + c * 32, sv + c * 32);
      tc_wait_ld();
      const int lim = pos - j * 128;   // keys past lim are in the future
      if (!__all_sync(0xffffffffu, lim >= 127)) {
#pragma unroll
        for (int x = 0; x < 128; ++x) sv[x] = x <= lim ? sv[x] : -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) m8[x] = sv[x];
#pragma unroll
      for (int x = 8; x < 128; ++x) m8[x & 7] = fmaxf(m8[x & 7], sv[x]);
      const float mblk = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * p.scale_log2;
      // a row whose maximum outgrew its reference rescales O (after PV(j-1))
      const bool grow = mblk > m_ref + kRescaleLog2;
      if (__any_sync(0xffffffffu, grow && j > 0)) {
        if (!(ok = mbar_wait(pvdone, (j - 1) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        const float a = grow ? fast_exp2(m_ref - mblk) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + lane_off + c * 32, ov);
          tc_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] *= a;
          tmem_st32(tO + lane_off + c * 32, ov);
        }
        tc_wait_st();
        l *= a;
      }
      if (grow) m_ref = mblk;
      float l8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) l8[x] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float e0 = fast_exp2(fmaf(sv[c * 32 + x], p.scale_log2, -m_ref));
          const float e1 = fast_exp2(fmaf(sv[c * 32 + x + 1], p.scale_log2, -m_ref));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
          const uint32_t w = *reinterpret_cast<uint32_t*>(&h2);
          pk[x >> 1] = w;
          l8[(x >> 1) & 7] += __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
        }
        tmem_st16(sbuf + c * 16, pk);
      }
      l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&pfull[st]);
    }
    // epilogue: after the last PV, O / l -> bf16 (PV(nblk-3) is known to be done,
    // so the parity waits for nblk-2 and then nblk-1 are unambiguous)
    if (ok && nblk >= 2) ok = mbar_wait(pvdone, (nblk - 2) & 1, abort_flag, p.err);
    if (ok && mbar_wait(pvdone, (nblk - 1) & 1, abort_flag, p.err)) {
      tc_fence_after();
      const float il = 1.f / l;
      const long long orow = (static_cast<long long>(b) * p.T + (valid ? t : t_last)) * p.H +
                             g * p.r + head;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(tO + lane_off + c * 32, ov);
        tc_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + orow * D + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            __nv_bfloat162 h0 = __floats2bfloat162_rn(ov[8 * x] * il, ov[8 * x + 1] * il);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(ov[8 * x + 2] * il, ov[8 * x + 3] * il);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[8 * x + 4] * il, ov[8 * x + 5] * il);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(ov[8 * x + 6] * il, ov[8 * x + 7] * il);
            dst[x] = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
          }
        }
      }
      if (valid && p.lse) p.lse[orow] = (m_ref + log2f(l)) / kLog2e;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch(const msa_shape& s, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   uint16_t* o, float* lse, const DevCtx* ctx, cudaStream_t st) {
  const int r = s.n_q_heads / s.n_kv_heads;
  DenseParams p{};
  p.o = o;
  p.lse = lse;
  p.err = ctx->err;
  p.T = s.seq_q;
  p.N = s.seq_kv;
  p.H = s.n_q_heads;
  p.G = s.n_kv_heads;
  p.r = r;
  p.q_off = s.q_offset;
  p.tpt = 128 / r;
  p.ntile = static_cast<int>(ceil_div(s.seq_q, p.tpt));
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
  CUtensorMap tq, tk, tv;
  const uint64_t dq[2] = {static_cast<uint64_t>(D),
                          static_cast<uint64_t>(s.batch) * s.seq_q * s.n_q_heads};
  const uint64_t sq[1] = {static_cast<uint64_t>(D) * 2};
  const uint32_t bq[2] = {64, static_cast<uint32_t>(r)};
  const uint64_t dk[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(s.seq_kv),
                          static_cast<uint64_t>(s.batch) * s.n_kv_heads};
  const uint64_t sk[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(s.seq_kv) * D * 2};
  const uint32_t bk[3] = {64, 128, 1};
  if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = DenseSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(dense_prefill_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(s.batch) * s.n_kv_heads * p.ntile;
  {
    ProfScope ps_("dense_prefill", st);
    dense_prefill_kernel<D><<<static_cast<unsigned>(grid), kThreads, smem, st>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dense_prefill(const msa_shape& s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, uint16_t* o, float* lse, cudaStream_t st) {
  const DevCtx* ctx = device_ctx();
  if (!ctx) return cudaErrorInitializationError;
  return s.head_dim == 128 ? launch<128>(s, q, k, v, o, lse, ctx, st)
                           : launch<64>(s, q, k, v, o, lse, ctx, st);
}

}  // namespace msa

namespace msa {
cudaError_t set_wait_limit_dense(uint64_t ns) { return set_wait_limit_here(ns); }
}  // namespace msa
