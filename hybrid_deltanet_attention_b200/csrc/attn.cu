// Causal GQA attention of a prefill pass on the sm_100a tensor cores, flash style: for each
// (128-query tile, query head) work item a CTA walks the cached keys in tiles of 64, keeps the scores of
// the current tile in tensor memory, turns them into probabilities with an online softmax in
// registers, and accumulates O = P V in tensor memory. No score or probability matrix
// leaves the chip; tiles above the diagonal are never computed.
//
// The math is that of the HN megakernel post's attention (QKV, RoPE, causal softmax,
// output projection); the queries arrive roped and scaled by 1/sqrt(D) as fp32, split into
// bf16 high and low parts (about 16 bits of their significand), the keys and values are the
// bf16 cache entries. Per key tile j:
//   S   = Q_hi K^T + Q_lo K^T            (tcgen05, M = 128, N = 64, K = D, into TMEM)
//   m_j = max(m, rowmax(S)); P = exp(S - m) masked above the diagonal; l += rowsum(P)
//   O   = O + P_hi V + P_lo V            (tcgen05, M = 128, N = D, K = 64, into TMEM)
// The running maximum m is only raised (and O, l rescaled by exp(m_old - m_new)) when a
// tile's maximum exceeds it by more than kRescaleAt; otherwise the stale maximum is kept,
// so every probability is at most e^kRescaleAt and the result O / l is the same softmax.
//
// The kernel is persistent: one CTA per SM takes items from a counter, the longest key
// ranges first (the last query tile of every head, then the one before, ...), so the causal
// imbalance evens out across the SMs; between items the CTA drains and re-arms its barriers.
// Roles (192 threads): warp 0 lane 0 issues the TMA loads (Q once, then K and V^T tiles),
// warp 1 lane 0 issues the MMAs, warps 2..5 (one TMEM lane quarter each, one query row per
// thread) run the softmax and write O / l. Every wait has a time limit; on expiry the CTA
// latches an error bit and winds down.
#include <algorithm>
#include <cstdint>
#include <cuda.h>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "tc.cuh"

namespace mk {

namespace {

constexpr int kFM = 128;                 // queries per CTA (TMEM lanes)
constexpr int kFN = 64;                  // keys per tile
constexpr int kFThreads = 192;
constexpr float kRescaleAt = 8.0f;       // natural log units
constexpr uint64_t kFlashWaitNs = 1000000000ull;
constexpr int kQBlk = kFM * 64 * 2;      // one 64-wide K block of 128 query rows: 16 KB
constexpr int kKBlk = kFN * 64 * 2;      // one 64-wide D block of 64 keys: 8 KB

// Shared-memory layout for head dim D (a multiple of 64 up to 256): Q high and low parts
// [D / 64 blocks][128][64], K [D / 64][64][64], V^T [D][64], P high and low parts [128][64].
template <int D>
struct FlashLayout {
  static constexpr int kNB = D / 64;
  static constexpr int kOffQhi = 0;
  static constexpr int kOffQlo = kOffQhi + kNB * kQBlk;
  static constexpr int kOffK = kOffQlo + kNB * kQBlk;
  static constexpr int kOffVt = kOffK + kNB * kKBlk;
  static constexpr int kOffPhi = kOffVt + D * 64 * 2;
  static constexpr int kOffPlo = kOffPhi + kFM * 64 * 2;
  static constexpr int kOffBars = kOffPlo + kFM * 64 * 2;
  static constexpr int kSmem = kOffBars + 256 + 1024;   // + barriers, + 1024-byte alignment slack
  // TMEM columns: O [0, D), S buffers [D, D + 64) and [D + 64, D + 128)
  static constexpr uint32_t kColO = 0, kColS = D;
  static constexpr uint32_t kTmemCols = D + 2 * kFN <= 256 ? 256 : 512;
};

struct FlashBars {
  uint64_t q_full, k_full, k_empty, v_full, v_empty, p_full, p_empty;
  uint64_t s_full[2], s_empty[2];
  uint32_t tmem;
  int abort;
  int item;   // the work item this CTA runs next
};
static_assert(sizeof(FlashBars) <= 256, "barriers fit their slot");


__device__ __forceinline__ bool fwait(FlashBars* fb, uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_wait(bar, parity, &fb->abort, kFlashWaitNs)) return true;
  if (!fb->abort) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
  fb->abort = 1;
  return false;
}

template <int D>
__global__ void __launch_bounds__(kFThreads, 1)
    attn_flash_kernel(const __grid_constant__ CUtensorMap tq_hi, const __grid_constant__ CUtensorMap tq_lo,
                      const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tvt,
                      const int* __restrict__ posp, int off, int T, int Hq, int Hkv, int max_ctx, float* __restrict__ out,
                      long long ldo, int* items, int* err) {
  using Lay = FlashLayout<D>;
  constexpr int kNB = Lay::kNB;
  constexpr int kOffQhi = Lay::kOffQhi, kOffQlo = Lay::kOffQlo, kOffK = Lay::kOffK, kOffVt = Lay::kOffVt;
  constexpr int kOffPhi = Lay::kOffPhi, kOffPlo = Lay::kOffPlo;
  constexpr uint32_t kColO = Lay::kColO, kColS = Lay::kColS, kTmemCols = Lay::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FlashBars* fb = reinterpret_cast<FlashBars*>(smem + Lay::kOffBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile_q = (T + kFM - 1) / kFM;
  const int n_items = ntile_q * Hq;
  const int pos0 = *posp + off;

  if (threadIdx.x == 0) {
    fb->abort = 0;
    tc::prefetch_tensormap(&tq_hi);
    tc::prefetch_tensormap(&tq_lo);
    tc::prefetch_tensormap(&tk);
    tc::prefetch_tensormap(&tvt);
  }
  if (warp == 0) {
    tc::tmem_alloc(&fb->tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = fb->tmem;

  for (;;) {
  if (threadIdx.x == 0) {   // next item; the barriers start a fresh sequence (nothing is pending)
    fb->item = fb->abort ? n_items : atomicAdd(items, 1);
    mbar_init(&fb->q_full, 1);
    mbar_init(&fb->k_full, 1);
    mbar_init(&fb->k_empty, 1);
    mbar_init(&fb->v_full, 1);
    mbar_init(&fb->v_empty, 1);
    mbar_init(&fb->p_full, 4);
    mbar_init(&fb->p_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&fb->s_full[b], 1);
      mbar_init(&fb->s_empty[b], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const int item = fb->item;
  if (item >= n_items) break;
  const int qt = ntile_q - 1 - item / Hq;   // the longest key ranges first
  const int h = item % Hq, g = h / (Hq / Hkv);
  const int m0 = qt * kFM;
  // keys 0 .. pos0 + (last valid query of the tile)
  const int nkeys = pos0 + min(m0 + kFM, T);
  const int nt = (nkeys + kFN - 1) / kFN;

  if (warp == 0) {
    if (lane == 0) {   // ---- TMA producer
      bool ok = true;
      mbar_arrive_expect_tx(&fb->q_full, 2 * kNB * kQBlk);
      for (int kb = 0; kb < kNB; ++kb) {
        tc::tma_load_2d(smem + kOffQhi + kb * kQBlk, &tq_hi, h * D + kb * 64, m0, &fb->q_full);
        tc::tma_load_2d(smem + kOffQlo + kb * kQBlk, &tq_lo, h * D + kb * 64, m0, &fb->q_full);
      }
      for (int j = 0; j < nt && ok; ++j) {
        if (j > 0 && !(ok = fwait(fb, &fb->k_empty, (j - 1) & 1, err))) break;   // S(j-1) read K(j-1)
        mbar_arrive_expect_tx(&fb->k_full, kNB * kKBlk);
        for (int kb = 0; kb < kNB; ++kb)
          tc::tma_load_2d(smem + kOffK + kb * kKBlk, &tk, kb * 64, g * max_ctx + j * kFN, &fb->k_full);
        if (j > 0 && !(ok = fwait(fb, &fb->v_empty, (j - 1) & 1, err))) break;   // PV(j-1) read V(j-1)
        mbar_arrive_expect_tx(&fb->v_full, D * 64 * 2);
        tc::tma_load_2d(smem + kOffVt, &tvt, j * kFN, g * D, &fb->v_full);
      }
      int never = 0;   // let the last copies land before the CTA ends (bounded)
      if (nt > 0) {
        mbar_wait(&fb->k_full, (nt - 1) & 1, &never, kFlashWaitNs / 5);
        mbar_wait(&fb->v_full, (nt - 1) & 1, &never, kFlashWaitNs / 5);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {   // ---- MMA issuer
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kFM, kFN);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(kFM, D);
      bool ok = fwait(fb, &fb->q_full, 0, err);
      tc::fence_after_sync();
      auto issue_s = [&](int j) -> bool {   // S(j) = Q K(j)^T into S buffer j & 1
        const int b = j & 1;
        if (!fwait(fb, &fb->k_full, j & 1, err)) return false;
        if (j >= 2 && !fwait(fb, &fb->s_empty[b], ((j >> 1) - 1) & 1, err)) return false;
        tc::fence_after_sync();
        const uint32_t ds = tmem + kColS + static_cast<uint32_t>(b * kFN);
        for (int kb = 0; kb < kNB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = tc::desc_kmajor_sw128(smem + kOffK + kb * kKBlk + kk * 32);
            tc::mma_bf16(ds, tc::desc_kmajor_sw128(smem + kOffQhi + kb * kQBlk + kk * 32), bd, idesc_s,
                         (kb | kk) ? 1u : 0u);
            tc::mma_bf16(ds, tc::desc_kmajor_sw128(smem + kOffQlo + kb * kQBlk + kk * 32), bd, idesc_s, 1u);
          }
        }
        tc::mma_commit(&fb->k_empty);
        tc::mma_commit(&fb->s_full[b]);
        return true;
      };
      if (ok && nt > 0) ok = issue_s(0);
      for (int j = 0; j < nt && ok; ++j) {
        if (j + 1 < nt && !(ok = issue_s(j + 1))) break;
        if (!(ok = fwait(fb, &fb->p_full, j & 1, err))) break;
        if (!(ok = fwait(fb, &fb->v_full, j & 1, err))) break;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // O += P V over the tile's 64 keys
          const uint64_t bd = tc::desc_kmajor_sw128(smem + kOffVt + kk * 32);
          tc::mma_bf16(tmem + kColO, tc::desc_kmajor_sw128(smem + kOffPhi + kk * 32), bd, idesc_o,
                       (j > 0 || kk) ? 1u : 0u);
          tc::mma_bf16(tmem + kColO, tc::desc_kmajor_sw128(smem + kOffPlo + kk * 32), bd, idesc_o, 1u);
        }
        tc::mma_commit(&fb->v_empty);
        tc::mma_commit(&fb->p_empty);
      }
    }
  } else {   // ---- softmax and epilogue: warps 2..5, thread = query row
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int qpos = pos0 + m0 + r;   // position of this row's query
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    uint8_t* phi = smem + kOffPhi;
    uint8_t* plo = smem + kOffPlo;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      const bool okw = mbar_wait(&fb->s_full[b], (j >> 1) & 1, &fb->abort, kFlashWaitNs);
      if (!__all_sync(0xffffffffu, okw) || fb->abort) {
        if (!okw && lane == 0) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
        fb->abort = 1;
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float s[kFN];
#pragma unroll
      for (int c = 0; c < kFN; c += 16) tc::tmem_ld16(tmem + lane_base + kColS + b * kFN + c, s + c);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&fb->s_empty[b]);   // the S buffer may be overwritten
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kFN; ++c) {
        if (j * kFN + c > qpos) s[c] = -INFINITY;   // causal mask (also keys past the pass)
        mx = fmaxf(mx, s[c]);
      }
      // P's shared memory is free and O is up to date once PV(j-1) has completed
      const bool okp = (j == 0) || mbar_wait(&fb->p_empty, (j - 1) & 1, &fb->abort, kFlashWaitNs);
      if (!__all_sync(0xffffffffu, okp) || fb->abort) {
        if (!okp && lane == 0) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
        fb->abort = 1;
        ok = false;
        break;
      }
      tc::fence_after_sync();
      if (j == 0) {
        m_used = mx;   // key 0 is visible to every query, so mx is finite
      } else {
        // raise the running maximum of the rows whose tile maximum passed it by more than
        // kRescaleAt: rescale their O and l. The TMEM loads and stores are warp-collective,
        // so the whole warp walks O whenever one of its rows needs it (factor 1 elsewhere).
        const bool raise = mx > m_used + kRescaleAt;
        if (__any_sync(0xffffffffu, raise)) {
          const float f = raise ? __expf(m_used - mx) : 1.0f;
          l *= f;
#pragma unroll 1
          for (int c = 0; c < D; c += 16) {
            float o[16];
            tc::tmem_ld16(tmem + lane_base + kColO + c, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] *= f;
            tc::tmem_st16(tmem + lane_base + kColO + c, o);
          }
          if (raise) m_used = mx;
        }
      }
      // P = exp(S - m) as bf16 high and low parts, K-major 128-byte-swizzled rows
      uint8_t* rh = phi + r * 128;
      uint8_t* rl = plo + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < kFN / 8; ++c8) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = __expf(s[c8 * 8 + 2 * i] - m_used), p1 = __expf(s[c8 * 8 + 2 * i + 1] - m_used);
          l += p0 + p1;
          const uint16_t h0 = f_to_bf16(p0), h1 = f_to_bf16(p1);
          hw[i] = h0 | (static_cast<uint32_t>(h1) << 16);
          lw[i] = f_to_bf16(p0 - bf16_to_f(h0)) | (static_cast<uint32_t>(f_to_bf16(p1 - bf16_to_f(h1))) << 16);
        }
        const int chunk = (c8 ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(rh + chunk) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(rl + chunk) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      tc::fence_proxy_async_smem();   // the tensor cores read P next
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&fb->p_full);
    }
    // O / l once the last PV has completed
    if (ok && nt > 0) {
      const bool okw = mbar_wait(&fb->p_empty, (nt - 1) & 1, &fb->abort, kFlashWaitNs);
      if (!okw && lane == 0) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
      if (__all_sync(0xffffffffu, okw)) {
        tc::fence_after_sync();
        const float inv = 1.0f / l;
        const int t = m0 + r;
        float* orow = out + static_cast<long long>(t) * ldo + static_cast<long long>(h) * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          float o[16];
          tc::tmem_ld16(tmem + lane_base + kColO + c, o);
          if (t < T) {
            float4* d4 = reinterpret_cast<float4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv,
                                                            o[4 * i + 3] * inv);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();   // the item is done in every role (O read out, copies landed)
  tc::fence_after_sync();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_flash_d(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mk_, const CUtensorMap& mvt,
                           const int* posp, int off, int T, int Hq, int Hkv, int max_ctx, float* out, long long ldo,
                           int* items, int* err, cudaStream_t s) {
  static std::atomic<uint64_t> attr_set{0};   // per device
  const cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(attn_flash_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FlashLayout<D>::kSmem);
  });
  if (e != cudaSuccess) return e;
  const int n_items = (T + kFM - 1) / kFM * Hq;
  int dev = 0, sms = 0;
  cudaError_t e2 = cudaGetDevice(&dev);
  if (e2 == cudaSuccess) e2 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e2 != cudaSuccess) return e2;
  e2 = cudaMemsetAsync(items, 0, sizeof(int), s);
  if (e2 != cudaSuccess) return e2;
  attn_flash_kernel<D><<<std::min(n_items, sms), kFThreads, FlashLayout<D>::kSmem, s>>>(
      mqh, mql, mk_, mvt, posp, off, T, Hq, Hkv, max_ctx, out, ldo, items, err);
  return cudaGetLastError();
}

}  // namespace

bool attn_flash_supported(int D) { return D == 64 || D == 128 || D == 256; }

// Causal attention of the T queries of a prefill pass (roped, pre-scaled, as bf16 high / low
// parts q_hi, q_lo [T][Hq * D]) over the keys 0 .. pos0 + t of one layer's cache: K rows
// k [Hkv][max_ctx][D] bf16 and V^T vt [Hkv][D][nk] bf16 (zero past the pass's last key), for
// D in {64, 128, 256}. out [T][ldo] fp32 gets O of head h at columns h * D. pos0 = *posp + off
// on the device; the key range is bounded by the host with nk (a multiple of 64, >= pos0 + T).
cudaError_t launch_attn_flash(const uint16_t* q_hi, const uint16_t* q_lo, const uint16_t* k, const uint16_t* vt,
                              const int* posp, int off, int T, int Hq, int Hkv, int D, int max_ctx, long long nk,
                              float* out, long long ldo, int* items, int* err, cudaStream_t s) {
  if (!attn_flash_supported(D) || T <= 0 || Hq % Hkv || nk % 64 || ldo % 4 || (reinterpret_cast<uintptr_t>(out) & 15) ||
      !items)
    return cudaErrorInvalidValue;
  CUtensorMap mqh, mql, mk_, mvt;
  const long long qd = static_cast<long long>(Hq) * D;
  if (!tensor_map_bf16(&mqh, q_hi, T, qd, qd * 2, kFM) || !tensor_map_bf16(&mql, q_lo, T, qd, qd * 2, kFM) ||
      !tensor_map_bf16(&mk_, k, static_cast<long long>(Hkv) * max_ctx, D, 2LL * D, kFN) ||
      !tensor_map_bf16(&mvt, vt, static_cast<long long>(Hkv) * D, nk, 2 * nk, D))
    return cudaErrorInvalidValue;
  if (D == 256) return launch_flash_d<256>(mqh, mql, mk_, mvt, posp, off, T, Hq, Hkv, max_ctx, out, ldo, items, err, s);
  if (D == 128) return launch_flash_d<128>(mqh, mql, mk_, mvt, posp, off, T, Hq, Hkv, max_ctx, out, ldo, items, err, s);
  return launch_flash_d<64>(mqh, mql, mk_, mvt, posp, off, T, Hq, Hkv, max_ctx, out, ldo, items, err, s);
}

}  // namespace mk
