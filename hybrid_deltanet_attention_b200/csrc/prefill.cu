// Batched prefill: a prompt's tokens go through every layer together, the projections
// as tensor-core GEMMs (gemm.cu), the DeltaNet mixer in its chunked (WY) form, the
// attention mixer causally over the KV cache (attn.cu for 64+ tokens). The last token's
// logits and the next token then come from its residual row (mk_prefill_tail).
//
// Per layer, for T tokens at positions pos0 .. pos0+T-1 (activations fp32 in HBM; every
// GEMM input is written as bf16 high/low parts):
//   x = RMSNorm(h)                          rms_split
//   DeltaNet: z = x W_in^T                  linear
//             conv + SiLU, q/k L2 norms,    dn_prep_v4, conv_history_update
//             log a = -softplus(alpha), b = sigmoid(beta)
//             chunked delta rule            wy_prep_tc / wy_prep_fast (per chunk and head),
//                                           wy_state_tc / wy_state_fast (per head and row group)
//   attention: z = x W_in^T                 linear
//             RoPE, K/V into the cache      at_prep
//             causal softmax attention      attn_flash_kernel (64+ tokens), attn_prefill
//   h += o W_out^T                          gate_split (with the output gate), linear (accumulate)
//   x = RMSNorm(h); g|u = x [W_gate|W_up]^T; h += (SiLU(g) u) W_down^T
#include <algorithm>
#include <cmath>
#include <string>

#include <cuda_fp16.h>

#include "../../include/mk.h"
#include "dev.cuh"
#include "mk_internal.h"
#include "mk_model.h"
#include "tc.cuh"

namespace mk {
namespace {

constexpr int kPT = 256;    // threads of the row kernels
constexpr int kPrepMaxConv = 4;   // causal conv width limit (checked at load)

// Threads of a row kernel: wide CTAs when a pass has few rows (verify, short tails).
inline int rms_threads(int T) { return T < 64 ? 1024 : kPT; }

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < static_cast<int>(blockDim.x >> 5)) ? red[l] : 0.f;
  return warp_sum(t);
}

// Four consecutive values (i a multiple of 4) as bf16 high / low parts, 8-byte stores.
__device__ __forceinline__ void put_split4(uint16_t* hi, uint16_t* lo, long long i, float4 v) {
  const float a[4] = {v.x, v.y, v.z, v.w};
  uint16_t h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    h[q] = f_to_bf16(a[q]);
    l[q] = f_to_bf16(a[q] - bf16_to_f(h[q]));
  }
  *reinterpret_cast<uint2*>(hi + i) = make_uint2(h[0] | (static_cast<uint32_t>(h[1]) << 16),
                                                 h[2] | (static_cast<uint32_t>(h[3]) << 16));
  *reinterpret_cast<uint2*>(lo + i) = make_uint2(l[0] | (static_cast<uint32_t>(l[1]) << 16),
                                                 l[2] | (static_cast<uint32_t>(l[3]) << 16));
}

__device__ __forceinline__ void put_split(uint16_t* hi, uint16_t* lo, long long i, float v) {
  const uint16_t h = f_to_bf16(v);
  hi[i] = h;
  lo[i] = f_to_bf16(v - bf16_to_f(h));
}

// h[t] = E[tok[t]] (bf16 -> fp32). An out-of-range id latches MK_DEVERR_BAD_TOKEN and
// gives a zero row.
__global__ void embed_rows(const int32_t* __restrict__ tok, int T, const uint16_t* __restrict__ embed, int lde, int H,
                           int V, float* __restrict__ h, int* err) {
  const int t = blockIdx.x;
  const int id = tok[t];
  const bool ok = id >= 0 && id < V;
  if (!ok && threadIdx.x == 0) atomicOr(err, MK_DEVERR_BAD_TOKEN);
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    h[static_cast<long long>(t) * H + i] = ok ? bf16_to_f(embed[static_cast<long long>(id) * lde + i]) : 0.f;
}

// x[t] = h[t] / sqrt(mean(h[t]^2) + eps) * gamma, written as bf16 high/low parts.
__global__ void rms_split(const float* __restrict__ h, int H, const uint16_t* __restrict__ gamma, float eps,
                          uint16_t* __restrict__ xhi, uint16_t* __restrict__ xlo) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* row = h + static_cast<long long>(t) * H;
  float ss = 0.f;   // H is a multiple of 4: float4 rows
  for (int i = 4 * threadIdx.x; i < H; i += 4 * blockDim.x) {
    const float4 v = *reinterpret_cast<const float4*>(row + i);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
  for (int i = 4 * threadIdx.x; i < H; i += 4 * blockDim.x) {
    const float4 v = *reinterpret_cast<const float4*>(row + i);
    const uint2 gw = *reinterpret_cast<const uint2*>(gamma + i);
    put_split4(xhi, xlo, static_cast<long long>(t) * H + i,
               make_float4(v.x * inv * bf16lo(gw.x), v.y * inv * bf16hi(gw.x), v.z * inv * bf16lo(gw.y),
                           v.w * inv * bf16hi(gw.y)));
  }
}

// h[t] = E[tok[t]] for 4-bit embedding rows (w = d sc q - dmin m per 32-weight sub-block).
__global__ void embed_rows_q4(const int32_t* __restrict__ tok, int T, const uint8_t* __restrict__ embed, int rb,
                              int H, int V, float* __restrict__ h, int* err) {
  const int t = blockIdx.x;
  const int id = tok[t];
  const bool ok = id >= 0 && id < V;
  if (!ok && threadIdx.x == 0) atomicOr(err, MK_DEVERR_BAD_TOKEN);
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    float v = 0.f;
    if (ok) {
      const uint8_t* blk = embed + static_cast<long long>(id) * rb + (i >> 8) * 144;
      const int e = i & 255, jb = e >> 5, w = e & 31;
      const uint32_t dd = *reinterpret_cast<const uint32_t*>(blk);
      const uint64_t lo = static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 4)) |
                          (static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 8)) << 32);
      const uint64_t hi = static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 8)) |
                          (static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 12)) << 32);
      const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(dd & 0xFFFFu))) *
                       static_cast<float>(static_cast<uint32_t>(lo >> (6 * jb)) & 63u);
      const float mn = __half2float(__ushort_as_half(static_cast<unsigned short>(dd >> 16))) *
                       static_cast<float>(static_cast<uint32_t>(hi >> (16 + 6 * jb)) & 63u);
      const uint32_t q = (blk[16 + 16 * jb + (w & 15)] >> (4 * (w >> 4))) & 15u;
      v = fmaf(sc, static_cast<float>(q), -mn);
    }
    h[static_cast<long long>(t) * H + i] = v;
  }
}

// C[t][n] (+)= sum_k X[t][k] W[n][k] with 4-bit rows W (Q4_K-style 144-byte super-blocks of
// 256 weights along k: fp16 d, dmin; 6-bit sub-block scales sc_j and mins m_j; 4-bit codes
// q, w = d sc_j q - dmin m_j) for up to 8 tokens per CTA, on the tensor cores with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate): the 32 weights of a sub-block enter as the
// exact bf16 values 128 + q, the tokens' activations as their bf16 high and low parts, so
//   sum_k w_k x_k = d sc_j (D_j - 128 X_j) - dmin m_j X_j,   D_j = sum_k (128 + q_k) x_k,
// with X_j = sum_k x_k over the sub-block taken by the same MMA against a tile of ones.
// A warp owns 32 rows (two m16 groups) and a slice of super-blocks (grid.y splits K when
// the rows alone leave the GPU idle; partial sums go to a workspace and are reduced in a
// fixed order); its rows stream through a private cp.async ring of 3 super-blocks.
// Token tile: grid.z (8 tokens each).
constexpr int kQ4Depth = 2;
__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// bytes [b0, b1] of a code pair -> bf16x2 (128 + q(b0), 128 + q(b1)) of the low (hi4 = 0) or
// high (hi4 = 1) nibbles
__device__ __forceinline__ uint32_t q4_pair_bf16(uint32_t spread, int hi4) {
  return ((hi4 ? (spread >> 4) : spread) & 0x000F000Fu) | 0x43004300u;
}

__global__ void __launch_bounds__(128, 5) q4_linear_mma(const uint16_t* __restrict__ xhi, const uint16_t* __restrict__ xlo,
                                                     int ldx, const uint8_t* __restrict__ W, long long ldw,
                                                     float* __restrict__ out, long long ldo, int T, int N, int K,
                                                     int sb_per_split, int accumulate) {
  constexpr int DEP = kQ4Depth, CH = 144 / 16, RPW = 32;
  extern __shared__ __align__(16) uint8_t q4m[];   // per warp: [DEP][32 rows][144]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  uint8_t* ring = q4m + warp * DEP * RPW * 144;
  const int n0 = blockIdx.x * 128 + warp * RPW;
  const int nsb = K >> 8;
  const int sbA = blockIdx.y * sb_per_split, sbB = min(nsb, sbA + sb_per_split);
  const int t0 = blockIdx.z * 8;
  const bool tok_ok = t0 + g < T;   // this lane's B column (token t0 + g)
  const uint16_t* xh = xhi + static_cast<long long>(tok_ok ? t0 + g : 0) * ldx + 2 * c;
  const uint16_t* xl = xlo + static_cast<long long>(tok_ok ? t0 + g : 0) * ldx + 2 * c;
  const uint8_t* rowp[CH];   // the 16-byte pieces this lane copies: i = lane + 32 m of 32 rows x 9
  int rowo[CH];
#pragma unroll
  for (int m = 0; m < CH; ++m) {
    const int i = lane + 32 * m, r = i / CH, ch = i % CH;
    rowp[m] = W + static_cast<long long>(min(n0 + r, N - 1)) * ldw + ch * 16;
    rowo[m] = r * 144 + ch * 16;
  }
  auto issue = [&](int sb) {
    if (sb < sbB) {
      uint8_t* slot = ring + ((sb - sbA) % DEP) * RPW * 144;
#pragma unroll
      for (int m = 0; m < CH; ++m) cp_async16(slot + rowo[m], rowp[m] + static_cast<long long>(sb) * 144, 16u);
    }
    cp_async_commit();
  };
  if (n0 < N) {
#pragma unroll
    for (int p = 0; p < DEP - 1; ++p) issue(sbA + p);
  }
  float acc[2][4];
#pragma unroll
  for (int gr = 0; gr < 2; ++gr)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[gr][i] = 0.f;
  const uint32_t ones = 0x3F803F80u;   // bf16 1.0, 1.0
  for (int sb = sbA; sb < sbB && n0 < N; ++sb) {
    issue(sb + DEP - 1);
    cp_async_wait<DEP - 1>();
    __syncwarp();
    const uint8_t* slot = ring + ((sb - sbA) % DEP) * RPW * 144;
    // my rows: rr = 0..3 -> row 16 (rr >> 1) + 8 (rr & 1) + g of the warp's 32
    const uint8_t* rb[4];
    uint4 hd[4];
    float dsc[4], dmn[4];   // the super-block's fp16 d and dmin of my 4 rows, once per super-block
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      rb[rr] = slot + ((rr >> 1) * 16 + (rr & 1) * 8 + g) * 144;
      hd[rr] = *reinterpret_cast<const uint4*>(rb[rr]);
      dsc[rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd[rr].x & 0xFFFFu)));
      dmn[rr] = __half2float(__ushort_as_half(static_cast<unsigned short>(hd[rr].x >> 16)));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // codes of sub-block j: bytes (2c, 2c+1) and (2c+8, 2c+9) of each row, spread to [b0, 0, b1, 0]
      uint32_t sp[4][2];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const uint32_t w0 = *reinterpret_cast<const uint16_t*>(rb[rr] + 16 + 16 * j + 2 * c);
        const uint32_t w1 = *reinterpret_cast<const uint16_t*>(rb[rr] + 16 + 16 * j + 2 * c + 8);
        sp[rr][0] = __byte_perm(w0, 0u, 0x4140);
        sp[rr][1] = __byte_perm(w1, 0u, 0x4140);
      }
      float dq[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}}, dx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // k-step: weights 16 h .. 16 h + 15 of the sub-block
        const int kb = sb * 256 + 32 * j + 16 * h;
        uint32_t bh0 = 0u, bh1 = 0u, bl0 = 0u, bl1 = 0u;
        if (tok_ok) {
          bh0 = *reinterpret_cast<const uint32_t*>(xh + kb); bh1 = *reinterpret_cast<const uint32_t*>(xh + kb + 8);
          bl0 = *reinterpret_cast<const uint32_t*>(xl + kb); bl1 = *reinterpret_cast<const uint32_t*>(xl + kb + 8);
        }
#pragma unroll
        for (int gr = 0; gr < 2; ++gr) {
          const uint32_t a0 = q4_pair_bf16(sp[2 * gr][0], h), a1 = q4_pair_bf16(sp[2 * gr + 1][0], h);
          const uint32_t a2 = q4_pair_bf16(sp[2 * gr][1], h), a3 = q4_pair_bf16(sp[2 * gr + 1][1], h);
          mma_bf16_16816(dq[gr], a0, a1, a2, a3, bh0, bh1);
          mma_bf16_16816(dq[gr], a0, a1, a2, a3, bl0, bl1);
        }
        mma_bf16_16816(dx, ones, ones, ones, ones, bh0, bh1);
        mma_bf16_16816(dx, ones, ones, ones, ones, bl0, bl1);
      }
      // scales of sub-block j for my 4 rows, then acc += s (D - 128 X) - mn X; the 6-bit
      // fields become floats through the exponent field (2^23 + v is exact), not a conversion
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const uint64_t lo = static_cast<uint64_t>(hd[rr].y) | (static_cast<uint64_t>(hd[rr].z) << 32);
        const uint64_t hi = static_cast<uint64_t>(hd[rr].z) | (static_cast<uint64_t>(hd[rr].w) << 32);
        const uint32_t scb = static_cast<uint32_t>(lo >> (6 * j)) & 63u;
        const uint32_t mmb = static_cast<uint32_t>(hi >> (16 + 6 * j)) & 63u;
        const float s = dsc[rr] * (__uint_as_float(0x4B000000u | scb) - 8388608.0f);
        const float mn = dmn[rr] * (__uint_as_float(0x4B000000u | mmb) - 8388608.0f);
        const int gr = rr >> 1, i0 = 2 * (rr & 1);   // D rows g (i 0, 1) or g + 8 (i 2, 3); tokens 2c, 2c + 1
        const float cx = -(128.f * s + mn);
        acc[gr][i0] = fmaf(s, dq[gr][i0], fmaf(cx, dx[0], acc[gr][i0]));
        acc[gr][i0 + 1] = fmaf(s, dq[gr][i0 + 1], fmaf(cx, dx[1], acc[gr][i0 + 1]));
      }
    }
    __syncwarp();   // every lane is done with this slot before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();
  if (n0 >= N) return;
  // D layout: element i of group gr is row 16 gr + g + 8 (i >> 1), token 2c + (i & 1)
  float* dst = out;
  long long ld = ldo;
  bool add = accumulate != 0;
  if (gridDim.y > 1) {   // partial sums [split][T][N]
    dst = out + static_cast<long long>(blockIdx.y) * T * N;
    ld = N;
    add = false;
  }
#pragma unroll
  for (int gr = 0; gr < 2; ++gr)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = n0 + 16 * gr + g + 8 * (i >> 1), t = t0 + 2 * c + (i & 1);
      if (n < N && t < T) {
        float* p = dst + static_cast<long long>(t) * ld + n;
        *p = add ? *p + acc[gr][i] : acc[gr][i];
      }
    }
}

// C[t][n] (+)= sum_k X[t][k] W[n][k] for bf16 rows W and up to 8 tokens per CTA (few-token
// passes: verify, short tails), on mma.sync m16n8k16: W tiles as the A operand (ldmatrix from
// a per-warp cp.async ring of 64-wide K blocks, 16-byte pieces XOR-swizzled by row so the
// matrix loads are conflict-free), the tokens' bf16 high / low activation parts as B, fp32
// accumulation in registers. A warp owns 32 rows and a slice of K blocks (grid.y splits K;
// partials reduced by q4_split_reduce); grid.z walks 8-token tiles.
constexpr int kBfDepth = 4;
__global__ void __launch_bounds__(128, 3) bf16_linear_mma(const uint16_t* __restrict__ xhi,
                                                          const uint16_t* __restrict__ xlo, int ldx,
                                                          const uint8_t* __restrict__ W, long long ldw,
                                                          float* __restrict__ out, long long ldo, int T, int N, int K,
                                                          int kb_per_split, int accumulate) {
  constexpr int DEP = kBfDepth, RPW = 32, KB = 64;   // K block: 64 bf16 = 128 bytes per row
  extern __shared__ __align__(16) uint8_t bfm[];     // per warp: [DEP][32 rows][128 B]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  uint8_t* ring = bfm + warp * DEP * RPW * 128;
  const int n0 = blockIdx.x * 128 + warp * RPW;
  const int nkb = K / KB;
  const int kbA = blockIdx.y * kb_per_split, kbB = min(nkb, kbA + kb_per_split);
  const int t0 = blockIdx.z * 8;
  const bool tok_ok = t0 + g < T;
  const uint16_t* xh = xhi + static_cast<long long>(tok_ok ? t0 + g : 0) * ldx + 2 * c;
  const uint16_t* xl = xlo + static_cast<long long>(tok_ok ? t0 + g : 0) * ldx + 2 * c;
  // copies: 32 rows x 8 pieces of 16 bytes per K block, 8 per lane; piece p of row r lands at
  // r * 128 + 16 (p ^ (r & 7))
  const uint8_t* src[8];
  int dsto[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int i = lane + 32 * m, r = i >> 3, pc = i & 7;
    src[m] = W + static_cast<long long>(min(n0 + r, N - 1)) * ldw + pc * 16;
    dsto[m] = r * 128 + 16 * (pc ^ (r & 7));
  }
  auto issue = [&](int kb) {
    if (kb < kbB) {
      uint8_t* slot = ring + ((kb - kbA) % DEP) * RPW * 128;
#pragma unroll
      for (int m = 0; m < 8; ++m) cp_async16(slot + dsto[m], src[m] + static_cast<long long>(kb) * 128, 16u);
    }
    cp_async_commit();
  };
  if (n0 < N) {
#pragma unroll
    for (int p = 0; p < DEP - 1; ++p) issue(kbA + p);
  }
  float acc[2][4];
#pragma unroll
  for (int gr = 0; gr < 2; ++gr)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[gr][i] = 0.f;
  // ldmatrix.x4 addresses: lanes 0-15 rows 0..15 at k 0..7, lanes 16-31 rows 0..15 at k 8..15
  const int lr = lane & 15, lk = lane >> 4;
  for (int kb = kbA; kb < kbB && n0 < N; ++kb) {
    issue(kb + DEP - 1);
    cp_async_wait<DEP - 1>();
    __syncwarp();
    const uint8_t* slot = ring + ((kb - kbA) % DEP) * RPW * 128;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {   // 16-wide k steps
      const int kglob = kb * KB + 16 * ks;
      uint32_t bh0 = 0u, bh1 = 0u, bl0 = 0u, bl1 = 0u;   // padding tokens stay zero
      if (tok_ok) {
        bh0 = *reinterpret_cast<const uint32_t*>(xh + kglob);
        bh1 = *reinterpret_cast<const uint32_t*>(xh + kglob + 8);
        bl0 = *reinterpret_cast<const uint32_t*>(xl + kglob);
        bl1 = *reinterpret_cast<const uint32_t*>(xl + kglob + 8);
      }
#pragma unroll
      for (int gr = 0; gr < 2; ++gr) {
        const int r = 16 * gr + lr, pc = 2 * ks + lk;
        const uint32_t addr = smem_u32(slot + r * 128 + 16 * (pc ^ (r & 7)));
        uint32_t a0, a1, a2, a3;
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                     : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                     : "r"(addr));
        mma_bf16_16816(acc[gr], a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(acc[gr], a0, a1, a2, a3, bl0, bl1);
      }
    }
    __syncwarp();   // every lane is done with this slot before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();
  if (n0 >= N) return;
  float* dst = out;
  long long ld = ldo;
  bool add = accumulate != 0;
  if (gridDim.y > 1) {   // partial sums [split][T][N]
    dst = out + static_cast<long long>(blockIdx.y) * T * N;
    ld = N;
    add = false;
  }
#pragma unroll
  for (int gr = 0; gr < 2; ++gr)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = n0 + 16 * gr + g + 8 * (i >> 1), t = t0 + 2 * c + (i & 1);
      if (n < N && t < T) {
        float* p = dst + static_cast<long long>(t) * ld + n;
        *p = add ? *p + acc[gr][i] : acc[gr][i];
      }
    }
}

// out[t][n] (+)= sum over splits z of ws[z][t][n], in order of z.
__global__ void q4_split_reduce(const float* __restrict__ ws, int nz, int T, int N, float* __restrict__ out,
                                long long ldo, int accumulate) {
  const long long tot = static_cast<long long>(T) * N;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < tot;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int z = 0; z < nz; ++z) v += ws[static_cast<long long>(z) * tot + i];
    const long long t = i / N, n = i % N;
    float* p = out + t * ldo + n;
    *p = accumulate ? *p + v : v;
  }
}

// DeltaNet token prep. z[t] = [q~ k~ v~ (C channels) | alpha (Hd) | beta (Hd)].
// y[t] = [q/|q| (Hd dk) | k/|k| (Hd dk) | v (Hd dv) | log a (Hd) | b (Hd)] with the causal
// conv + SiLU over the C channels (inputs before pos0 come from the conv history ring,
// slot p mod W holding position p), log a = -softplus(alpha), b = sigmoid(beta).
__global__ void dn_prep(const float* __restrict__ z, int ldz, const int* __restrict__ posp, int off,
                        const float* __restrict__ ring, int W, int C, int Hd, int dk, const uint16_t* __restrict__ taps,
                        float* __restrict__ y, int ldy) {
  extern __shared__ float ys[];   // [C]
  __shared__ float nrm[2 * 64];
  const int t = blockIdx.x;
  const int pos0 = *posp + off;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < W; ++j) {
      const int s = t - (W - 1) + j;        // token index inside this batch
      float x;
      if (s >= 0) x = z[static_cast<long long>(s) * ldz + c];
      else {
        const int p = pos0 + s;             // absolute position
        x = p >= 0 ? ring[static_cast<long long>(p % W) * C + c] : 0.f;
      }
      acc = fmaf(bf16_to_f(taps[static_cast<long long>(c) * W + j]), x, acc);
    }
    ys[c] = siluf_(acc);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int vec = warp; vec < 2 * Hd; vec += nw) {     // q heads then k heads
    float ss = 0.f;
    for (int d = lane; d < dk; d += 32) ss += ys[vec * dk + d] * ys[vec * dk + d];
    ss = warp_sum(ss);
    if (lane == 0) nrm[vec] = 1.0f / sqrtf(ss + 1e-6f);
  }
  __syncthreads();
  float* yr = y + static_cast<long long>(t) * ldy;
  const int qk = 2 * Hd * dk;
  for (int c = threadIdx.x; c < C; c += blockDim.x) yr[c] = c < qk ? ys[c] * nrm[c / dk] : ys[c];
  for (int hh = threadIdx.x; hh < Hd; hh += blockDim.x) {
    const float al = z[static_cast<long long>(t) * ldz + C + hh];
    const float be = z[static_cast<long long>(t) * ldz + C + Hd + hh];
    yr[C + hh] = -(fmaxf(al, 0.f) + log1pf(expf(-fabsf(al))));
    yr[C + Hd + hh] = sigmoidf_(be);
  }
}

// The same with one warp per (8 consecutive tokens, 128-channel block) and four channels
// per lane (float4 loads of z, the ring and the outputs; C a multiple of 128, dk 64 or 128,
// row strides multiples of 4 floats). The lane keeps the conv window of its channels in
// registers and slides it over the warp's tokens (one new z row per token); the q / k norms
// reduce over the dk / 4 lanes of a head with shuffles. Block C / 128 holds the gates.
constexpr int kPrepTokensPerWarp = 8;
__global__ void __launch_bounds__(256) dn_prep_v4(const float* __restrict__ z, int ldz, int T,
                                                  const int* __restrict__ posp, int off, const float* __restrict__ ring,
                                                  int W, int C, int Hd, int dk, const uint16_t* __restrict__ taps,
                                                  float* __restrict__ y, int ldy) {
  constexpr int TPW = kPrepTokensPerWarp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = (blockIdx.x * 8 + warp) * TPW;
  if (tb >= T) return;
  const int te = min(T, tb + TPW);
  if (static_cast<int>(blockIdx.y) * 128 >= C) {   // gates
    for (int t = tb; t < te; ++t) {
      const float* zt = z + static_cast<long long>(t) * ldz;
      float* yr = y + static_cast<long long>(t) * ldy;
      for (int hh = lane; hh < Hd; hh += 32) {
        const float al = zt[C + hh], be = zt[C + Hd + hh];
        yr[C + hh] = -(fmaxf(al, 0.f) + log1pf(expf(-fabsf(al))));
        yr[C + Hd + hh] = sigmoidf_(be);
      }
    }
    return;
  }
  const int pos0 = *posp + off;
  const int c0 = blockIdx.y * 128 + 4 * lane;
  const bool qk = c0 < 2 * Hd * dk;   // warp-uniform: blocks are all q / k or all v channels
  // window of the last kPrepMaxConv input rows; tap j of a width-W conv sits at slot j + (4 - W)
  constexpr int MW = kPrepMaxConv;
  float tw[4][MW];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int j = 0; j < MW; ++j) {
      const int jj = j - (MW - W);
      tw[u][j] = jj >= 0 ? bf16_to_f(taps[static_cast<long long>(c0 + u) * W + jj]) : 0.f;
    }
  auto load = [&](int s) {   // input row s of the pass (negative: conv history)
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s >= 0) {
      v = *reinterpret_cast<const float4*>(z + static_cast<long long>(s) * ldz + c0);
    } else {
      const int p = pos0 + s;
      if (p >= 0) v = *reinterpret_cast<const float4*>(ring + static_cast<long long>(p % W) * C + c0);
    }
    return v;
  };
  float4 win[MW];   // win[j] = input row t - (MW - 1) + j
#pragma unroll
  for (int j = 0; j < MW - 1; ++j) win[j] = j >= MW - W ? load(tb - (MW - 1) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t = tb; t < te; ++t) {
    win[MW - 1] = load(t);
    float o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < MW; ++j) {
        const float xv = u == 0 ? win[j].x : (u == 1 ? win[j].y : (u == 2 ? win[j].z : win[j].w));
        acc = fmaf(tw[u][j], xv, acc);
      }
      o[u] = siluf_(acc);
    }
    if (qk) {   // L2 norm over the head (dk / 4 lanes, aligned)
      float ss = o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3];
      for (int m = dk / 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      const float nr = 1.0f / sqrtf(ss + 1e-6f);
#pragma unroll
      for (int u = 0; u < 4; ++u) o[u] *= nr;
    }
    *reinterpret_cast<float4*>(y + static_cast<long long>(t) * ldy + c0) = make_float4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int j = 0; j + 1 < MW; ++j) win[j] = win[j + 1];
  }
}

// The same on a (token, vector) grid: vector v < 2 Hd is one q or k head (conv + SiLU +
// L2 norm over its dk <= 128 channels), then blocks of 128 v channels, then the gates.
// Enough CTAs for a few-token pass (a verify pass has T = K + 1).
__global__ void __launch_bounds__(128) dn_prep_wide(const float* __restrict__ z, int ldz, const int* __restrict__ posp,
                                                    int off, const float* __restrict__ ring, int W, int C, int Hd, int dk,
                                                    int dv, const uint16_t* __restrict__ taps, float* __restrict__ y,
                                                    int ldy) {
  __shared__ float red[4];
  const int t = blockIdx.x, vec = blockIdx.y, tid = threadIdx.x;
  const int pos0 = *posp + off;
  const int nqk = 2 * Hd, nvb = (Hd * dv + 127) / 128;
  auto conv = [&](int c) -> float {
    float acc = 0.f;
    for (int j = 0; j < W; ++j) {
      const int s = t - (W - 1) + j;
      float x;
      if (s >= 0) x = z[static_cast<long long>(s) * ldz + c];
      else {
        const int p = pos0 + s;
        x = p >= 0 ? ring[static_cast<long long>(p % W) * C + c] : 0.f;
      }
      acc = fmaf(bf16_to_f(taps[static_cast<long long>(c) * W + j]), x, acc);
    }
    return siluf_(acc);
  };
  float* yr = y + static_cast<long long>(t) * ldy;
  if (vec < nqk) {
    const int c = vec * dk + tid;
    const float v = tid < dk ? conv(c) : 0.f;
    const float ss = warp_sum(v * v);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] + red[1] + red[2] + red[3] + 1e-6f);
    if (tid < dk) yr[c] = v * inv;
  } else if (vec < nqk + nvb) {
    const int c = 2 * Hd * dk + (vec - nqk) * 128 + tid;
    if (c < C) yr[c] = conv(c);
  } else {
    for (int hh = tid; hh < Hd; hh += blockDim.x) {
      const float al = z[static_cast<long long>(t) * ldz + C + hh];
      const float be = z[static_cast<long long>(t) * ldz + C + Hd + hh];
      yr[C + hh] = -(fmaxf(al, 0.f) + log1pf(expf(-fabsf(al))));
      yr[C + Hd + hh] = sigmoidf_(be);
    }
  }
}

// Conv history after the batch: the raw inputs of the last W-1 positions go to their ring slots.
__global__ void conv_history_update(const float* __restrict__ z, int ldz, int T, const int* __restrict__ posp, int off,
                                    float* __restrict__ ring, int W, int C) {
  const int m = blockIdx.y;                 // 0 .. W-2: position pos0 + T - 1 - m
  const int s = T - 1 - m;
  if (s < 0) return;
  const int p = *posp + off + s;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < C; c += gridDim.x * blockDim.x)
    ring[static_cast<long long>(p % W) * C + c] = z[static_cast<long long>(s) * ldz + c];
}

// Attention token prep: RoPE (half-split pairs (i, i + D/2), angle (pos0+t) * inv_freq_i)
// on the Hq query heads (then scaled by 1/sqrt(D)) and the Hkv key heads; keys and values
// appended to the bf16 cache at position pos0 + t.
__global__ void at_prep(const float* __restrict__ z, int ldz, const int* __restrict__ posp, int off,
                        const double* __restrict__ inv_freq, int Hq, int Hkv, int D, int gated, uint16_t* __restrict__ kc,
                        uint16_t* __restrict__ vc, int max_ctx, float* __restrict__ q, int ldq, int kv_rb, int kv_q8) {
  extern __shared__ float kvs[];   // 8-bit cache: the token's roped keys [Hkv][D], then values [Hkv][D]
  const int t = blockIdx.x, pos = *posp + off + t, half = D / 2;
  if (pos < 0 || pos >= max_ctx) return;    // capacity: latched by check_capacity
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float* zr = z + static_cast<long long>(t) * ldz;
  const int koff = Hq * D * (gated ? 2 : 1), voff = koff + Hkv * D;
  for (int idx = threadIdx.x; idx < (Hq + Hkv) * half; idx += blockDim.x) {
    const int hv = idx / half, i = idx % half;
    float cs, sn;
    rope_cs(static_cast<double>(pos) * inv_freq[i], cs, sn);
    if (hv < Hq) {
      const float x1 = zr[hv * D + i], x2 = zr[hv * D + i + half];
      q[static_cast<long long>(t) * ldq + hv * D + i] = (x1 * cs - x2 * sn) * scale;
      q[static_cast<long long>(t) * ldq + hv * D + i + half] = (x1 * sn + x2 * cs) * scale;
    } else {
      const int g = hv - Hq;
      const float x1 = zr[koff + g * D + i], x2 = zr[koff + g * D + i + half];
      if (kv_q8) {
        kvs[g * D + i] = x1 * cs - x2 * sn;
        kvs[g * D + i + half] = x1 * sn + x2 * cs;
      } else {
        const long long base = (static_cast<long long>(g) * max_ctx + pos) * D;
        kc[base + i] = f_to_bf16(x1 * cs - x2 * sn);
        kc[base + i + half] = f_to_bf16(x1 * sn + x2 * cs);
      }
    }
  }
  for (int idx = threadIdx.x; idx < Hkv * D; idx += blockDim.x) {
    const int g = idx / D, d = idx % D;
    if (kv_q8) kvs[Hkv * D + idx] = zr[voff + idx];
    else vc[(static_cast<long long>(g) * max_ctx + pos) * D + d] = f_to_bf16(zr[voff + idx]);
  }
  if (!kv_q8) return;
  __syncthreads();   // 8-bit rows: blocks of 32 entries, one warp per block
  const int nb = D / 32, lane = threadIdx.x & 31;
  for (int blk = threadIdx.x >> 5; blk < 2 * Hkv * nb; blk += blockDim.x >> 5) {
    const bool isv = blk >= Hkv * nb;
    const int b2 = blk - (isv ? Hkv * nb : 0), g = b2 / nb, jb = b2 % nb;
    uint8_t* row = reinterpret_cast<uint8_t*>(isv ? vc : kc) + (static_cast<size_t>(g) * max_ctx + pos) * kv_rb;
    unsigned short sbits;
    float back;
    const int qc = q8_block_lane(kvs[(isv ? Hkv * D : 0) + g * D + jb * 32 + lane], sbits, back);
    row[jb * 32 + lane] = static_cast<uint8_t>(static_cast<int8_t>(qc));
    if (lane == 0) reinterpret_cast<unsigned short*>(row + D)[jb] = sbits;
  }
}

// Rows [0, nrows) of one attention layer's 8-bit K and V, read back as bf16 into
// out [2][Hkv][max_ctx][D] for the attention kernels; rows past the pass's last key
// (device position) are written as zeros.
__global__ void kv_dequant_bf16(const uint8_t* __restrict__ kq, const uint8_t* __restrict__ vq, int Hkv, int D,
                                int max_ctx, int kv_rb, const int* __restrict__ posp, int last_off,
                                uint16_t* __restrict__ out) {
  const int r = blockIdx.x, g = blockIdx.y, which = blockIdx.z;
  const int last = min(*posp + last_off, max_ctx - 1);
  uint16_t* dst = out + ((static_cast<size_t>(which) * Hkv + g) * max_ctx + r) * D;
  const uint8_t* src = (which ? vq : kq) + (static_cast<size_t>(g) * max_ctx + r) * kv_rb;
  const unsigned short* sc = reinterpret_cast<const unsigned short*>(src + D);
  for (int d = threadIdx.x; d < D; d += blockDim.x)
    dst[d] = r <= last ? f_to_bf16(__half2float(__ushort_as_half(sc[d >> 5])) *
                                   static_cast<float>(static_cast<int8_t>(src[d])))
                       : static_cast<uint16_t>(0);
}

// x = o (* sigmoid(gate) when gate != null), as bf16 high/low parts [T][n].
__global__ void gate_split(const float* __restrict__ o, int ldo, const float* __restrict__ gate, int ldg, int n,
                           uint16_t* __restrict__ xhi, uint16_t* __restrict__ xlo) {
  const int t = blockIdx.x;   // n, ldo, ldg multiples of 4: float4 rows
  for (int i = 4 * (blockIdx.y * blockDim.x + threadIdx.x); i < n; i += 4 * gridDim.y * blockDim.x) {
    float4 v = *reinterpret_cast<const float4*>(o + static_cast<long long>(t) * ldo + i);
    if (gate) {
      const float4 g = *reinterpret_cast<const float4*>(gate + static_cast<long long>(t) * ldg + i);
      v.x *= sigmoidf_(g.x); v.y *= sigmoidf_(g.y); v.z *= sigmoidf_(g.z); v.w *= sigmoidf_(g.w);
    }
    put_split4(xhi, xlo, static_cast<long long>(t) * n + i, v);
  }
}

// act = SiLU(g) * u from gu[t] = [g (F) | u (F)], as bf16 high/low parts [T][F].
__global__ void act_split(const float* __restrict__ gu, int F, uint16_t* __restrict__ xhi, uint16_t* __restrict__ xlo) {
  const int t = blockIdx.x;   // F a multiple of 4: float4 rows
  const float* r = gu + static_cast<long long>(t) * 2 * F;
  for (int i = 4 * (blockIdx.y * blockDim.x + threadIdx.x); i < F; i += 4 * gridDim.y * blockDim.x) {
    const float4 g = *reinterpret_cast<const float4*>(r + i);
    const float4 u = *reinterpret_cast<const float4*>(r + F + i);
    put_split4(xhi, xlo, static_cast<long long>(t) * F + i,
               make_float4(siluf_(g.x) * u.x, siluf_(g.y) * u.y, siluf_(g.z) * u.z, siluf_(g.w) * u.w));
  }
}

// ------------------------------------------------------------------ chunked delta rule
// One head, one chunk of n <= 64 tokens (r = 0..n-1) with incoming state S0 [dv][dk]:
//   g_r = sum_{s<=r} log a_s,  gamma_r = e^{g_r},  dec_r = e^{g_{n-1} - g_r}
//   A[r][s] = b_r e^{g_r - g_s} (k_r . k_s)  (s < r, strictly lower triangular)
//   U = (I + A)^-1 diag(b) V,   W = (I + A)^-1 diag(b gamma) K
//   P[r][s] = e^{g_r - g_s} (q_r . k_s)  (s <= r)
// and then, with Delta = U - W S0^T (row r = the delta-rule update of token r),
//   o_r = gamma_r S0 q_r + sum_{s<=r} P[r][s] Delta_s,
//   S_n = gamma_{n-1} S0 + sum_r dec_r Delta_r k_r^T.
// Only differences g_r - g_s with s <= r are exponentiated, so every factor is <= 1.
constexpr int kChunk = 64;
constexpr int kRowGroup = 16;   // rows of S per CTA in the state pass

struct WyBufs {
  const float* y;   // dn_prep output, row stride ldy
  int ldy;
  float* u;         // [T][Hd dv]
  float* w;         // [T][Hd dk]
  float* p;         // [n_chunks][Hd][64][64]
  float* gam;       // [T][Hd]
  float* dec;       // [T][Hd]
  float* o;         // [T][Hd dv]
  int T, Hd, dk, dv;
  // verify passes (one chunk): keep g, k and the updates Delta, leave S untouched
  float* save_g;     // [T][Hd] or null
  float* save_k;     // [T][Hd dk] or null
  float* save_delta; // [T][Hd dv] or null
  int keep_state;
  // tensor-core state pass: bf16 operand images per (chunk, head), see WyImg; null = fp32 w, p
  uint8_t* img;
  int* err;          // device error word (tensor-core state pass)
};

// Operand images of one (chunk, head) for the tensor-core state pass: bf16 high and low
// parts of K-major, 128-byte-swizzled tiles (64 bf16 of K per 128-byte row, the layout a
// 128-byte-swizzled TMA load writes), so that one bulk copy stages each:
//   A1 [part][dk/64 K blocks][128 rows]: rows 0..63 gamma_r q_r, rows 64..127 w_r (K = dk)
//   P  [part][64 rows]:  P[r][s] (K = s)
//   KT [part][128 rows]: row j holds k_r[j] over r (K = r); rows j >= dk are zero
template <int DK>
struct WyImg {
  static constexpr uint32_t kA1 = 2u * (DK / 64) * 16384u;
  static constexpr uint32_t kP = 2u * 8192u;
  static constexpr uint32_t kKT = 2u * 16384u;
  static constexpr uint32_t kBytes = kA1 + kP + kKT;
};

// Eight floats as bf16 high parts (hi) and the bf16 of the remainders (lo).
__device__ __forceinline__ void split8_bf16(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint16_t h0 = f_to_bf16(v[2 * q]), h1 = f_to_bf16(v[2 * q + 1]);
    const uint16_t l0 = f_to_bf16(v[2 * q] - bf16_to_f(h0)), l1 = f_to_bf16(v[2 * q + 1] - bf16_to_f(h1));
    h[q] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
    l[q] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__global__ void __launch_bounds__(256) wy_prep(WyBufs b) {
  extern __shared__ float sm[];
  const int dk = b.dk, dv = b.dv, Hd = b.Hd;
  const int ch = blockIdx.x, h = blockIdx.y;
  const int t0 = ch * kChunk, n = min(kChunk, b.T - t0);
  const int kp = dk + 1, xw = dv + dk;
  float* K = sm;                       // [64][dk+1]
  float* Q = K + kChunk * kp;          // [64][dk+1]
  float* X = Q + kChunk * kp;          // [64][dv+dk]: right-hand sides, then U | W
  float* A = X + kChunk * xw;          // [64][65]
  float* g = A + kChunk * 65;          // [64]
  float* bb = g + kChunk;              // [64]
  const int qo = h * dk, ko = Hd * dk + h * dk, vo = 2 * Hd * dk + h * dv;
  const int C = 2 * Hd * dk + Hd * dv;
  for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
    const int r = idx / dk, j = idx % dk;
    const float* yr = b.y + static_cast<long long>(t0 + r) * b.ldy;
    K[r * kp + j] = r < n ? yr[ko + j] : 0.f;
    Q[r * kp + j] = r < n ? yr[qo + j] : 0.f;
  }
  if (threadIdx.x < kChunk) {
    const int r = threadIdx.x;
    const float* yr = b.y + static_cast<long long>(t0 + r) * b.ldy;
    g[r] = r < n ? yr[C + h] : 0.f;     // log a, summed below
    bb[r] = r < n ? yr[C + Hd + h] : 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 0.f;
    for (int r = 0; r < kChunk; ++r) {
      acc += g[r];
      g[r] = acc;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kChunk * xw; idx += blockDim.x) {
    const int r = idx / xw, j = idx % xw;
    float v = 0.f;
    if (r < n) {
      if (j < dv) v = bb[r] * b.y[static_cast<long long>(t0 + r) * b.ldy + vo + j];
      else v = bb[r] * expf(g[r]) * K[r * kp + (j - dv)];
    }
    X[r * xw + j] = v;
  }
  // A (strictly lower) and P (lower with the diagonal); P goes straight to global memory
  float* P = b.p + (static_cast<long long>(ch) * Hd + h) * kChunk * kChunk;
  for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) {
    const int r = idx / kChunk, s = idx % kChunk;
    float a = 0.f, pq = 0.f;
    if (s <= r && r < n) {
      float dkk = 0.f, dqk = 0.f;
      for (int j = 0; j < dk; ++j) {
        const float ks = K[s * kp + j];
        dkk = fmaf(K[r * kp + j], ks, dkk);
        dqk = fmaf(Q[r * kp + j], ks, dqk);
      }
      const float e = expf(g[r] - g[s]);
      if (s < r) a = bb[r] * e * dkk;
      pq = e * dqk;
    }
    A[r * 65 + s] = a;
    P[idx] = pq;
  }
  __syncthreads();
  // forward substitution (I + A) X = RHS; column j is owned by one thread
  for (int j = threadIdx.x; j < xw; j += blockDim.x) {
    for (int r = 1; r < n; ++r) {
      float acc = X[r * xw + j];
      for (int s = 0; s < r; ++s) acc = fmaf(-A[r * 65 + s], X[s * xw + j], acc);
      X[r * xw + j] = acc;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < n * xw; idx += blockDim.x) {
    const int r = idx / xw, j = idx % xw;
    if (j < dv) b.u[static_cast<long long>(t0 + r) * Hd * dv + h * dv + j] = X[r * xw + j];
    else b.w[static_cast<long long>(t0 + r) * Hd * dk + h * dk + (j - dv)] = X[r * xw + j];
  }
  if (threadIdx.x < n) {
    const int r = threadIdx.x;
    b.gam[static_cast<long long>(t0 + r) * Hd + h] = expf(g[r]);
    b.dec[static_cast<long long>(t0 + r) * Hd + h] = expf(g[n - 1] - g[r]);
    if (b.save_g) b.save_g[static_cast<long long>(t0 + r) * Hd + h] = g[r];
  }
  if (b.save_k) {
    for (int idx = threadIdx.x; idx < n * dk; idx += blockDim.x) {
      const int r = idx / dk, j = idx % dk;
      b.save_k[static_cast<long long>(t0 + r) * Hd * dk + h * dk + j] = K[r * kp + j];
    }
  }
}

// State pass over the chunks of one head for kRowGroup rows of S (rows are independent).
__global__ void __launch_bounds__(256) wy_state(WyBufs b, float* __restrict__ S /* this layer [Hd][dv][dk] */) {
  extern __shared__ float sm[];
  const int dk = b.dk, dv = b.dv, Hd = b.Hd;
  const int h = blockIdx.x, i0 = blockIdx.y * kRowGroup;
  const int kp = dk + 1;
  float* S0 = sm;                          // [16][dk+1]
  float* Wc = S0 + kRowGroup * kp;         // [64][dk+1]
  float* Qc = Wc + kChunk * kp;            // [64][dk+1]
  float* Kc = Qc + kChunk * kp;            // [64][dk]
  float* Pc = Kc + kChunk * dk;            // [64][65]
  float* Uc = Pc + kChunk * 65;            // [64][16]
  float* Dl = Uc + kChunk * kRowGroup;     // [64][17]
  float* gm = Dl + kChunk * 17;            // [64]
  float* dc = gm + kChunk;                 // [64]
  float* Sg = S + (static_cast<long long>(h) * dv + i0) * dk;
  for (int idx = threadIdx.x; idx < kRowGroup * dk; idx += blockDim.x)
    S0[(idx / dk) * kp + idx % dk] = Sg[idx];
  const int qo = h * dk, ko = Hd * dk + h * dk;
  const int nch = (b.T + kChunk - 1) / kChunk;
  const int ti = threadIdx.x % kRowGroup, tr = threadIdx.x / kRowGroup;   // (row of S, token group)
  for (int ch = 0; ch < nch; ++ch) {
    const int t0 = ch * kChunk, n = min(kChunk, b.T - t0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < kChunk * dk; idx += blockDim.x) {
      const int r = idx / dk, j = idx % dk;
      const bool in = r < n;
      const long long t = t0 + r;
      Wc[r * kp + j] = in ? b.w[t * Hd * dk + h * dk + j] : 0.f;
      Qc[r * kp + j] = in ? b.y[t * b.ldy + qo + j] : 0.f;
      Kc[r * dk + j] = in ? b.y[t * b.ldy + ko + j] : 0.f;
    }
    const float* P = b.p + (static_cast<long long>(ch) * Hd + h) * kChunk * kChunk;
    for (int idx = threadIdx.x; idx < kChunk * kChunk; idx += blockDim.x) Pc[(idx / kChunk) * 65 + idx % kChunk] = P[idx];
    for (int idx = threadIdx.x; idx < kChunk * kRowGroup; idx += blockDim.x) {
      const int r = idx / kRowGroup, i = idx % kRowGroup;
      Uc[idx] = r < n ? b.u[static_cast<long long>(t0 + r) * Hd * dv + h * dv + i0 + i] : 0.f;
    }
    if (threadIdx.x < kChunk) {
      const int r = threadIdx.x;
      gm[r] = r < n ? b.gam[static_cast<long long>(t0 + r) * Hd + h] : 0.f;
      dc[r] = r < n ? b.dec[static_cast<long long>(t0 + r) * Hd + h] : 0.f;
    }
    __syncthreads();
    // Delta = U - W S0^T
    for (int r = tr; r < kChunk; r += 256 / kRowGroup) {
      float acc = 0.f;
      for (int j = 0; j < dk; ++j) acc = fmaf(Wc[r * kp + j], S0[ti * kp + j], acc);
      Dl[r * 17 + ti] = Uc[r * kRowGroup + ti] - acc;
      if (b.save_delta && r < n) b.save_delta[static_cast<long long>(t0 + r) * Hd * dv + h * dv + i0 + ti] = Dl[r * 17 + ti];
    }
    __syncthreads();
    // o_r = gamma_r S0 q_r + sum_{s<=r} P[r][s] Delta_s
    for (int r = tr; r < n; r += 256 / kRowGroup) {
      float sq = 0.f;
      for (int j = 0; j < dk; ++j) sq = fmaf(Qc[r * kp + j], S0[ti * kp + j], sq);
      float acc = gm[r] * sq;
      for (int s = 0; s <= r; ++s) acc = fmaf(Pc[r * 65 + s], Dl[s * 17 + ti], acc);
      b.o[static_cast<long long>(t0 + r) * Hd * dv + h * dv + i0 + ti] = acc;
    }
    __syncthreads();
    if (b.keep_state) continue;
    // S0 <- gamma_{n-1} S0 + sum_r dec_r Delta_r k_r^T
    const float gl = gm[n - 1];
    for (int idx = threadIdx.x; idx < kRowGroup * dk; idx += blockDim.x) {
      const int i = idx / dk, j = idx % dk;
      float acc = gl * S0[i * kp + j];
      for (int r = 0; r < n; ++r) acc = fmaf(dc[r] * Dl[r * 17 + i], Kc[r * dk + j], acc);
      S0[i * kp + j] = acc;
    }
  }
  __syncthreads();
  if (b.keep_state) return;
  for (int idx = threadIdx.x; idx < kRowGroup * dk; idx += blockDim.x) Sg[idx] = S0[(idx / dk) * kp + idx % dk];
}

// Register-tiled versions of the two kernels above for dk = dv = 64 or 128: float4
// shared-memory traffic (rows padded by 4 floats: 16-byte aligned, conflict-free for the
// access patterns below), 4 x 4 output tiles per thread, and the forward substitution on
// a right-hand-side column held in registers.
// Forward substitution (I + A) X = RHS for the first CH rows of a chunk (CH >= n), column
// j of X held in registers; writes the U (j < DV) or W column.
template <int CH, int DK, int DV>
__device__ __forceinline__ void wy_fsub(const WyBufs& b, const float* K, const float* A, const float* g,
                                        const float* bb, int t0, int n, int h, int j, int vo) {
  constexpr int KP = DK + 4, AP = kChunk + 4;
  const int Hd = b.Hd;
  float x[CH];
#pragma unroll
  for (int r = 0; r < CH; ++r) {
    float v = 0.f;
    if (r < n) {
      v = (j < DV) ? b.y[static_cast<long long>(t0 + r) * b.ldy + vo + j] : expf(g[r]) * K[r * KP + (j - DV)];
      v *= bb[r];
    }
    x[r] = v;
  }
#pragma unroll
  for (int r = 1; r < CH; ++r) {
    float a0 = x[r], a1 = 0.f, a2 = 0.f, a3 = 0.f;   // four partial chains
#pragma unroll
    for (int s4 = 0; s4 < r; s4 += 4) {
      const float4 a4 = *reinterpret_cast<const float4*>(A + r * AP + s4);
      a0 = fmaf(-a4.x, x[s4], a0);
      if (s4 + 1 < r) a1 = fmaf(-a4.y, x[s4 + 1], a1);
      if (s4 + 2 < r) a2 = fmaf(-a4.z, x[s4 + 2], a2);
      if (s4 + 3 < r) a3 = fmaf(-a4.w, x[s4 + 3], a3);
    }
    x[r] = (a0 + a1) + (a2 + a3);
  }
#pragma unroll
  for (int r = 0; r < CH; ++r) {
    if (r < n) {
      if (j < DV) b.u[static_cast<long long>(t0 + r) * Hd * DV + h * DV + j] = x[r];
      else b.w[static_cast<long long>(t0 + r) * Hd * DK + h * DK + (j - DV)] = x[r];
    }
  }
}

template <int DK, int DV>
__global__ void __launch_bounds__(256) wy_prep_fast(WyBufs b) {
  constexpr int KP = DK + 4, AP = kChunk + 4, XW = DV + DK;
  static_assert(XW <= 256, "one right-hand-side column per thread");
  extern __shared__ float4 sm4[];
  float* K = reinterpret_cast<float*>(sm4);   // [64][KP]
  float* Q = K + kChunk * KP;                 // [64][KP]
  float* A = Q + kChunk * KP;                 // [64][AP]
  float* g = A + kChunk * AP;                 // [64]
  float* bb = g + kChunk;                     // [64]
  const int Hd = b.Hd, tid = threadIdx.x;
  const int ch = blockIdx.x, h = blockIdx.y;
  const int t0 = ch * kChunk, n = min(kChunk, b.T - t0);
  const int qo = h * DK, ko = Hd * DK + h * DK, vo = 2 * Hd * DK + h * DV;
  const int C = 2 * Hd * DK + Hd * DV;
  for (int idx = tid; idx < kChunk * DK / 4; idx += 256) {   // rows past the prompt read as zero
    const int r = idx / (DK / 4), j4 = idx % (DK / 4);
    const float* yr = b.y + static_cast<long long>(t0 + min(r, n - 1)) * b.ldy;
    const uint32_t nb = r < n ? 16u : 0u;
    cp_async16(K + r * KP + 4 * j4, yr + ko + 4 * j4, nb);
    cp_async16(Q + r * KP + 4 * j4, yr + qo + 4 * j4, nb);
  }
  if (tid < 2 * kChunk) {
    const int r = tid & (kChunk - 1);
    const float* yr = b.y + static_cast<long long>(t0 + min(r, n - 1)) * b.ldy;
    if (tid < kChunk) cp_async4(g + r, yr + C + h, r < n ? 4u : 0u);
    else cp_async4(bb + r, yr + C + Hd + h, r < n ? 4u : 0u);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  if (tid < 32) {   // inclusive prefix sum of log a over the chunk (two values per lane)
    float v0 = g[2 * tid], v1 = g[2 * tid + 1];
    v1 += v0;
    float run = v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float x = __shfl_up_sync(0xffffffffu, run, o);
      if (tid >= o) run += x;
    }
    const float before = run - v1;
    g[2 * tid] = before + v0;
    g[2 * tid + 1] = run;
  }
  __syncthreads();
  // A[r][s] = b_r e^{g_r - g_s} k_r.k_s (s < r),  P[r][s] = e^{g_r - g_s} q_r.k_s (s <= r)
  {
    const int rt = tid >> 4, st = tid & 15;
    float akk[4][4], aqk[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) akk[a][c] = aqk[a][c] = 0.f;
#pragma unroll 4
    for (int j = 0; j < DK; j += 4) {
      float4 kr[4], qr[4], ks[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        kr[a] = *reinterpret_cast<const float4*>(K + (rt + 16 * a) * KP + j);
        qr[a] = *reinterpret_cast<const float4*>(Q + (rt + 16 * a) * KP + j);
        ks[a] = *reinterpret_cast<const float4*>(K + (st + 16 * a) * KP + j);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          akk[a][c] += kr[a].x * ks[c].x + kr[a].y * ks[c].y + kr[a].z * ks[c].z + kr[a].w * ks[c].w;
          aqk[a][c] += qr[a].x * ks[c].x + qr[a].y * ks[c].y + qr[a].z * ks[c].z + qr[a].w * ks[c].w;
        }
    }
    float* P = b.p + (static_cast<long long>(ch) * Hd + h) * kChunk * kChunk;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = rt + 16 * a, s2 = st + 16 * c;
        const bool live = r < n;
        const float e = (s2 <= r && live) ? expf(g[r] - g[s2]) : 0.f;
        A[r * AP + s2] = (s2 < r) ? bb[r] * e * akk[a][c] : 0.f;
        P[r * kChunk + s2] = e * aqk[a][c];
      }
  }
  __syncthreads();
  // (I + A) X = [diag(b) V | diag(b gamma) K]: column j of X in registers
  if (tid < XW) {
    if (n <= 16) wy_fsub<16, DK, DV>(b, K, A, g, bb, t0, n, h, tid, vo);
    else wy_fsub<kChunk, DK, DV>(b, K, A, g, bb, t0, n, h, tid, vo);
  }
  if (tid < n) {
    b.gam[static_cast<long long>(t0 + tid) * Hd + h] = expf(g[tid]);
    b.dec[static_cast<long long>(t0 + tid) * Hd + h] = expf(g[n - 1] - g[tid]);
    if (b.save_g) b.save_g[static_cast<long long>(t0 + tid) * Hd + h] = g[tid];
  }
  if (b.save_k) {
    for (int idx = tid; idx < n * DK; idx += 256) {
      const int r = idx / DK, j = idx % DK;
      b.save_k[static_cast<long long>(t0 + r) * Hd * DK + h * DK + j] = K[r * KP + j];
    }
  }
}

// Inputs of one chunk are fetched with cp.async in three groups so that their L2 latency
// hides behind the previous phase: W, Q, U, gamma and the decay factors of chunk c+1 are
// issued once chunk c's Delta is formed, P of chunk c+1 once chunk c's outputs are written,
// and K of chunk c at the top of its own iteration (K is read last, by the state update).
template <int DK, int DV>
__global__ void __launch_bounds__(256) wy_state_fast(WyBufs b, float* __restrict__ S) {
  constexpr int KP = DK + 4, AP = kChunk + 4, RG = kRowGroup;
  extern __shared__ float4 sm4[];
  float* S0 = reinterpret_cast<float*>(sm4);  // [16][KP]
  float* Wc = S0 + RG * KP;                   // [64][KP]
  float* Qc = Wc + kChunk * KP;               // [64][KP]
  float* Kc = Qc + kChunk * KP;               // [64][KP]
  float* Pc = Kc + kChunk * KP;               // [64][AP]
  float* DT = Pc + kChunk * AP;               // [16][AP]  Delta^T
  float* Uc = DT + RG * AP;                   // [64][16]
  float* gmb = Uc + kChunk * RG;              // [2][64] gamma, by chunk parity
  float* dcb = gmb + 2 * kChunk;              // [2][64] e^{g_last - g_r}, by chunk parity
  const int Hd = b.Hd, tid = threadIdx.x;
  const int h = blockIdx.x, i0 = blockIdx.y * RG;
  float* Sg = S + (static_cast<long long>(h) * DV + i0) * DK;
  const int qo = h * DK, ko = Hd * DK + h * DK;
  const int nch = (b.T + kChunk - 1) / kChunk;
  const bool upd = !b.keep_state;
  // W, Q, U, gamma, decay of chunk c (rows past the prompt read as zero)
  auto fetch_wqu = [&](int c) {
    const int t0 = c * kChunk, n = min(kChunk, b.T - t0);
    for (int idx = tid; idx < kChunk * DK / 4; idx += 256) {
      const int r = idx / (DK / 4), j4 = idx % (DK / 4);
      const long long t = t0 + min(r, n - 1);
      const uint32_t nb = r < n ? 16u : 0u;
      cp_async16(Wc + r * KP + 4 * j4, b.w + t * Hd * DK + h * DK + 4 * j4, nb);
      cp_async16(Qc + r * KP + 4 * j4, b.y + t * b.ldy + qo + 4 * j4, nb);
    }
    {
      const int r = tid >> 2, q4 = tid & 3;   // 64 rows x 4 float4 of U
      const long long t = t0 + min(r, n - 1);
      cp_async16(Uc + r * RG + 4 * q4, b.u + t * Hd * DV + h * DV + i0 + 4 * q4, r < n ? 16u : 0u);
    }
    if (tid < 2 * kChunk) {
      const int r = tid & (kChunk - 1);
      const long long t = t0 + min(r, n - 1);
      const uint32_t nb = r < n ? 4u : 0u;
      if (tid < kChunk) cp_async4(gmb + (c & 1) * kChunk + r, b.gam + t * Hd + h, nb);
      else cp_async4(dcb + (c & 1) * kChunk + r, b.dec + t * Hd + h, nb);
    }
  };
  auto fetch_p = [&](int c) {   // P is stored for all 64 rows of every chunk
    const float* P = b.p + (static_cast<long long>(c) * Hd + h) * kChunk * kChunk;
    for (int idx = tid; idx < kChunk * kChunk / 4; idx += 256) {
      const int r = idx / (kChunk / 4), s4 = idx % (kChunk / 4);
      cp_async16(Pc + r * AP + 4 * s4, P + r * kChunk + 4 * s4, 16u);
    }
  };
  for (int idx = tid; idx < RG * DK / 4; idx += 256) {
    const int i = idx / (DK / 4), j4 = idx % (DK / 4);
    cp_async16(S0 + i * KP + 4 * j4, Sg + i * DK + 4 * j4, 16u);
  }
  fetch_wqu(0);
  cp_async_commit();
  fetch_p(0);
  cp_async_commit();
  const int rg = tid >> 4, ti = tid & 15;       // rows rg + 16 a of the chunk, column ti of the group
  for (int ch = 0; ch < nch; ++ch) {
    const int t0 = ch * kChunk, n = min(kChunk, b.T - t0);
    const float* gm = gmb + (ch & 1) * kChunk;
    const float* dc = dcb + (ch & 1) * kChunk;
    __syncthreads();   // Kc is free: the previous state update is done
    if (upd) {
      for (int idx = tid; idx < kChunk * DK / 4; idx += 256) {
        const int r = idx / (DK / 4), j4 = idx % (DK / 4);
        const long long t = t0 + min(r, n - 1);
        cp_async16(Kc + r * KP + 4 * j4, b.y + t * b.ldy + ko + 4 * j4, r < n ? 16u : 0u);
      }
    }
    cp_async_commit();
    cp_async_wait<2>();   // W, Q, U, gamma, decay of this chunk (and S0 before the first)
    __syncthreads();
    // Delta = U - W S0^T and Q S0^T, rows rg + 16 a, column ti
    float dw[4] = {0.f, 0.f, 0.f, 0.f}, dq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int j = 0; j < DK; j += 4) {
      const float4 s4 = *reinterpret_cast<const float4*>(S0 + ti * KP + j);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float4 w4 = *reinterpret_cast<const float4*>(Wc + (rg + 16 * a) * KP + j);
        const float4 q4 = *reinterpret_cast<const float4*>(Qc + (rg + 16 * a) * KP + j);
        dw[a] += w4.x * s4.x + w4.y * s4.y + w4.z * s4.z + w4.w * s4.w;
        dq[a] += q4.x * s4.x + q4.y * s4.y + q4.z * s4.z + q4.w * s4.w;
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = rg + 16 * a;
      const float d = Uc[r * RG + ti] - dw[a];
      DT[ti * AP + r] = d;
      if (b.save_delta && r < n) b.save_delta[static_cast<long long>(t0 + r) * Hd * DV + h * DV + i0 + ti] = d;
    }
    cp_async_wait<1>();   // P of this chunk
    __syncthreads();      // Delta and P visible; W, Q, U free
    if (ch + 1 < nch) fetch_wqu(ch + 1);
    cp_async_commit();
    // o_r = gamma_r (Q S0^T)_r + sum_s P[r][s] Delta_s   (P is zero above the diagonal)
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = rg + 16 * a;
      float acc = gm[r] * dq[a];
#pragma unroll 4
      for (int s = 0; s < kChunk; s += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(Pc + r * AP + s);
        const float4 d4 = *reinterpret_cast<const float4*>(DT + ti * AP + s);
        acc += p4.x * d4.x + p4.y * d4.y + p4.z * d4.z + p4.w * d4.w;
      }
      if (r < n) b.o[static_cast<long long>(t0 + r) * Hd * DV + h * DV + i0 + ti] = acc;
    }
    __syncthreads();      // P and the unscaled Delta are consumed
    if (ch + 1 < nch) fetch_p(ch + 1);
    cp_async_commit();
    if (upd) {
      for (int idx = tid; idx < RG * kChunk; idx += 256) {   // Delta_r scaled by e^{g_{n-1} - g_r}
        const int i = idx / kChunk, r = idx % kChunk;
        DT[i * AP + r] *= dc[r];
      }
    }
    cp_async_wait<2>();   // K of this chunk
    __syncthreads();
    if (!upd) continue;
    // S0 <- gamma_{n-1} S0 + sum_r (dec_r Delta_r) k_r^T: row ti2, float4 columns jq, jq + 16, ...
    const float gl = gm[n - 1];
    const int ti2 = tid >> 4, jq = tid & 15;
#pragma unroll
    for (int c = 0; c < DK / 64; ++c) {
      const int j = 4 * jq + 64 * c;
      float4 acc = *reinterpret_cast<const float4*>(S0 + ti2 * KP + j);
      acc.x *= gl; acc.y *= gl; acc.z *= gl; acc.w *= gl;
#pragma unroll 4
      for (int r = 0; r < kChunk; r += 4) {
        const float4 d4 = *reinterpret_cast<const float4*>(DT + ti2 * AP + r);
        const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 k4 = *reinterpret_cast<const float4*>(Kc + (r + u) * KP + j);
          acc.x = fmaf(dd[u], k4.x, acc.x);
          acc.y = fmaf(dd[u], k4.y, acc.y);
          acc.z = fmaf(dd[u], k4.z, acc.z);
          acc.w = fmaf(dd[u], k4.w, acc.w);
        }
      }
      *reinterpret_cast<float4*>(S0 + ti2 * KP + j) = acc;   // only this thread touches these elements here
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (b.keep_state) return;
  for (int idx = tid; idx < RG * DK / 4; idx += 256) {
    const int i = idx / (DK / 4), j4 = idx % (DK / 4);
    *reinterpret_cast<float4*>(Sg + i * DK + 4 * j4) = *reinterpret_cast<const float4*>(S0 + i * KP + 4 * j4);
  }
}

// State pass on the tensor cores (chunks of 64, two or more per pass). CTA (head h, rows
// i0 .. i0 + 15 of S), 128 threads; thread t owns TMEM lane t. Per chunk, with every
// product taken as hi*hi + hi*lo + lo*hi of bf16 parts into fp32 (tcgen05.mma, M = 128,
// N = 16, K = 16):
//   A: D1 = [gamma Q; W] S0^T                   (lanes 0..63: gamma Q S0^T, 64..127: W S0^T)
//   Delta = U - W S0^T (lanes 64..127), written as bf16 tiles Delta^T, (dec Delta)^T
//   C: D3 = gamma_last S0^T + K^T (dec Delta)   (S^T accumulates in TMEM across chunks;
//                                                committed on its own barrier)
//   B: D1[0..63] += P Delta                     (o; the P tile's M = 128 operand spans the
//                                                next 64 rows of the image, whose products
//                                                land in lanes 64..127, which are not read)
// then S1 = D3 is copied to the S0 operand tile and pre-scaled by the next chunk's
// gamma_last. Only A, Delta and C lie on the chain from one chunk's state to the next: D1 is
// double-buffered, so B and the store of o run while the next chunk's A is under way.
// Operand images arrive by bulk copies: A1 of the next chunk as soon as phase A has consumed
// it, P and K^T two chunks ahead (double buffer); U and the decay factors by cp.async. Every
// wait has a time limit; on expiry the CTA latches an error and stops.
struct WyTcBars {
  uint64_t a1, pk[2], mma, mmas;
  uint32_t tmem;
  int abort;
};
constexpr uint64_t kWyWaitNs = 1000000000ull;

// Chunk-local part of the chunked delta rule with its three contractions on the tensor cores
// (one CTA of 128 threads per (chunk, head); writes what wy_prep_fast writes for the
// tensor-core state pass: U, gamma, the decay factors and the operand images A1, P, K^T).
//   (1) [K; Q] K^T  (M = 128 rows: the chunk's keys, then its queries; N = 64 keys; K = dk)
//       gives k_r.k_s and q_r.k_s in TMEM; A = strictly-lower(b_r e^{g_r-g_s} k_r.k_s) and
//       P = lower(e^{g_r-g_s} q_r.k_s) are formed from them in registers.
//   (2) T = (I + A)^-1 by forward substitution on the CUDA cores (one column per thread, 64
//       columns: a quarter of the work of substituting all dv + dk right-hand sides).
//   (3) U^T = (diag(b) V)^T T^T and W^T = (diag(b gamma) K)^T T^T (M = 128 feature rows, N = 64
//       tokens, K = 64 tokens), i.e. [U | W] = T [diag(b) V | diag(b gamma) K].
// Every product takes bf16 high and low parts (hi.hi + hi.lo + lo.hi, fp32 accumulation),
// which keeps about 16 bits of each operand. Shared memory (~98 KB, two CTAs per SM): the
// [K; Q] image (64 KB; once (1) has consumed it, it holds the columns of T, then the V and K
// images of step 3, then the W rows of the A1 image on their way out) and a
// 33 KB region that first stages the fp32 key rows, then the query rows (one bulk round trip
// each), and then holds the T image and A.
struct WyPrepTcLayout {
  static constexpr uint32_t kImg = 0;                    // [K;Q] image | later V and K images, 64 KB
  static constexpr uint32_t kStage = 65536;              // fp32 rows [64][128] | later T image + A
  static constexpr uint32_t kT = kStage;                 // T image: [hi, lo][64 rows][128 B]
  static constexpr uint32_t kA = kStage + 16384;         // fp32 A [64][68]
  static constexpr uint32_t kG = kA + 64 * 68 * 4;       // g, b, gamma = e^g, b gamma: [64] each
  static constexpr uint32_t kBar = kG + 4 * 64 * 4;      // mbarrier, TMEM base, abort flag
  static constexpr uint32_t kBytes = kBar + 32;
};
static_assert(WyPrepTcLayout::kG - WyPrepTcLayout::kStage >= 64 * 128 * 4, "the staging region holds 64 fp32 rows");
constexpr size_t kWyPrepTcSmem = WyPrepTcLayout::kBytes + 1024;   // + alignment slack

// bf16 high / low parts of v, written at (row, k) of a K-major 128-byte-swizzled tile pair
// (the low part tile `lo_off` bytes after the high part).
__device__ __forceinline__ void put_bf16_pair(uint8_t* tile, uint32_t lo_off, uint32_t row, uint32_t k, float v) {
  const uint16_t hi = f_to_bf16(v);
  const uint32_t off = tc::sw128_offset(row, k);
  *reinterpret_cast<uint16_t*>(tile + off) = hi;
  *reinterpret_cast<uint16_t*>(tile + lo_off + off) = f_to_bf16(v - bf16_to_f(hi));
}

template <int DK, int DV>
__global__ void __launch_bounds__(128, 2) wy_prep_tc(WyBufs b) {
  static_assert(DK == DV && (DK == 64 || DK == 128), "dk = dv = 64 or 128");
  using Lyt = WyPrepTcLayout;
  using I = WyImg<DK>;
  constexpr int KB = DK / 64, AP = kChunk + 4;
  extern __shared__ uint8_t wyp_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wyp_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* KQ = sm + Lyt::kImg;     // [hi: KB blocks][lo: KB blocks] of 128 rows x 128 B
  uint8_t* VI = sm + Lyt::kImg;     // step 3: diag(b) V image [hi][lo] of 128 rows x 128 B (K = tokens)
  uint8_t* KI = VI + 32768;         //         diag(b gamma) K image, same shape
  float* stg = reinterpret_cast<float*>(sm + Lyt::kStage);   // [64][DK] fp32 rows
  uint8_t* TI = sm + Lyt::kT;       // T image [hi][lo] of 64 rows x 128 B (K = tokens)
  float* A = reinterpret_cast<float*>(sm + Lyt::kA);
  float* g = reinterpret_cast<float*>(sm + Lyt::kG);
  float* bb = g + kChunk;
  float* gm = bb + kChunk;    // gamma_r = e^{g_r}
  float* bgm = gm + kChunk;   // b_r gamma_r
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lyt::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lyt::kBar + 8);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + Lyt::kBar + 12);
  const int Hd = b.Hd, tid = threadIdx.x, warp = tid >> 5;
  const int ch = blockIdx.x, h = blockIdx.y;
  const int t0 = ch * kChunk, n = min(kChunk, b.T - t0);
  const int qo = h * DK, ko = Hd * DK + h * DK, vo = 2 * Hd * DK + h * DV;
  const int C = 2 * Hd * DK + Hd * DV;
  uint8_t* img = b.img + (static_cast<size_t>(ch) * Hd + h) * I::kBytes;
  uint8_t* a1 = img;
  uint8_t* pimg = img + I::kA1;
  uint8_t* kt = pimg + I::kP;
  // fp32 rows [64][DK] of the chunk at column offset `col` of y into the staging region (rows
  // past the prompt read as zero)
  auto stage_rows = [&](int col) {
    for (int idx = tid; idx < kChunk * DK / 4; idx += 128) {
      const int r = idx / (DK / 4), j4 = idx % (DK / 4);
      const float* yr = b.y + static_cast<long long>(t0 + min(r, n - 1)) * b.ldy + col + 4 * j4;
      cp_async16(stg + r * DK + 4 * j4, yr, r < n ? 16u : 0u);
    }
  };

  stage_rows(ko);
  {   // gates of the chunk
    const int r = tid & (kChunk - 1);
    const float* yr = b.y + static_cast<long long>(t0 + min(r, n - 1)) * b.ldy;
    if (tid < kChunk) cp_async4(g + r, yr + C + h, r < n ? 4u : 0u);
    else cp_async4(bb + r, yr + C + Hd + h, r < n ? 4u : 0u);
  }
  cp_async_commit();
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tslot, 256);
    tc::tmem_relinquish();
  }
  cp_async_wait<0>();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tslot;
  const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
  if (tid < 32) {   // inclusive prefix sum of log a over the chunk (two values per lane)
    float v0 = g[2 * tid], v1 = g[2 * tid + 1];
    v1 += v0;
    float run = v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float x = __shfl_up_sync(0xffffffffu, run, o);
      if (tid >= o) run += x;
    }
    const float before = run - v1;
    g[2 * tid] = before + v0;
    g[2 * tid + 1] = run;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = 2 * tid + u;
      gm[r] = expf(g[r]);
      bgm[r] = bb[r] * gm[r];
    }
  }
  // ---- key rows: rows 0..63 of the [K; Q] image, and the K^T image (row j: k_r[j] over the
  // chunk's r; rows j >= dk zero, global)
#pragma unroll 1
  for (int idx = tid; idx < kChunk * (DK / 8); idx += 128) {
    const int r = idx / (DK / 8), c8 = idx % (DK / 8), kb = c8 >> 3, c = c8 & 7;
    uint4 hv, lv;
    split8_bf16(stg + r * DK + 8 * c8, hv, lv);
    const uint32_t off = static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4);
    *reinterpret_cast<uint4*>(KQ + kb * 16384 + off) = hv;
    *reinterpret_cast<uint4*>(KQ + (KB + kb) * 16384 + off) = lv;
  }
  {
    const int j = tid;
#pragma unroll 2
    for (int c = 0; c < 8; ++c) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = j < DK ? stg[(8 * c + u) * DK + j] : 0.f;
      uint4 hv, lv;
      split8_bf16(v, hv, lv);
      const uint32_t off = static_cast<uint32_t>(j) * 128u + ((static_cast<uint32_t>(c) ^ (j & 7u)) << 4);
      *reinterpret_cast<uint4*>(kt + off) = hv;
      *reinterpret_cast<uint4*>(kt + 16384 + off) = lv;
    }
  }
  __syncthreads();   // the staging region is free; gamma is published
  // ---- query rows: rows 64..127 of the [K; Q] image and the gamma Q rows of the A1 image
  stage_rows(qo);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
#pragma unroll 1
  for (int idx = tid; idx < kChunk * (DK / 8); idx += 128) {
    const int r = idx / (DK / 8), c8 = idx % (DK / 8), kb = c8 >> 3, c = c8 & 7;
    const int row = kChunk + r;
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = stg[r * DK + 8 * c8 + u];
    uint4 hv, lv;
    split8_bf16(v, hv, lv);
    const uint32_t off = static_cast<uint32_t>(row) * 128u + ((static_cast<uint32_t>(c) ^ (row & 7u)) << 4);
    *reinterpret_cast<uint4*>(KQ + kb * 16384 + off) = hv;
    *reinterpret_cast<uint4*>(KQ + (KB + kb) * 16384 + off) = lv;
    const float gr = gm[r];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] *= gr;
    split8_bf16(v, hv, lv);
    const uint32_t offq = static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4);
    *reinterpret_cast<uint4*>(a1 + kb * 16384 + offq) = hv;
    *reinterpret_cast<uint4*>(a1 + (KB + kb) * 16384 + offq) = lv;
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // ---- (1) D_A = [K; Q] K^T  (TMEM columns 0..63)
  if (tid == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(128, 64);
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t dh = tc::desc_kmajor_sw128(KQ + kb * 16384 + kk * 32);
        const uint64_t dl = tc::desc_kmajor_sw128(KQ + (KB + kb) * 16384 + kk * 32);
        tc::mma_bf16(tbase, dh, dh, idesc, (kb | kk) ? 1u : 0u);
        tc::mma_bf16(tbase, dh, dl, idesc, 1u);
        tc::mma_bf16(tbase, dl, dh, idesc, 1u);
      }
    tc::mma_commit(bar);
  }
  if (tid < n) {
    b.gam[static_cast<long long>(t0 + tid) * Hd + h] = gm[tid];
    b.dec[static_cast<long long>(t0 + tid) * Hd + h] = expf(g[n - 1] - g[tid]);
  }
  if (!mbar_wait(bar, 0, abort, kWyWaitNs)) {
    if (!*abort) atomicOr(b.err, MK_DEVERR_PIPE_TIMEOUT);
    *abort = 1;
  }
  tc::fence_after_sync();
  // ---- A (lanes 0..63) into shared memory, P (lanes 64..127) as the P image (global)
  {
    const int r = tid & (kChunk - 1);
    const bool isq = tid >= kChunk;
    const float gr = g[r], br = bb[r];
    const bool live = r < n;
    // decay factors e^{g_r - g_s} <= 1 (s <= r) by the fast exponential: relative error ~2^-21
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      float d[16];
      tc::tmem_ld16(tbase + lane_off + 16 * q, d);
      if (!isq) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int s = 16 * q + u;
          A[r * AP + s] = (s < r && live) ? br * __expf(gr - g[s]) * d[u] : 0.f;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int s = 16 * q + u;
          d[u] = (s <= r && live) ? __expf(gr - g[s]) * d[u] : 0.f;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint4 hv, lv;
          split8_bf16(d + 8 * hh, hv, lv);
          const uint32_t c = 2 * q + hh;
          const uint32_t off = static_cast<uint32_t>(r) * 128u + ((c ^ (r & 7u)) << 4);
          *reinterpret_cast<uint4*>(pimg + off) = hv;
          *reinterpret_cast<uint4*>(pimg + 8192 + off) = lv;
        }
      }
    }
  }
  __syncthreads();   // A complete; the [K; Q] image has been consumed
  if (*abort) {
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
    return;
  }
  // ---- (2) T = (I + A)^-1, one column per thread (threads 0..63), by blocks of 16 rows:
  // x_B = (e_j)_B - sum_{C < B} A_{BC} x_C, then the unit-lower 16 x 16 diagonal block. The
  // columns are kept in shared memory (the [K; Q] image is consumed), so the loop over the
  // earlier blocks stays a loop and the code stays small.
  float* X = reinterpret_cast<float*>(sm + Lyt::kImg);   // [64 rows][64 columns] fp32
  if (tid < kChunk) {
    const int j = tid;
#pragma unroll 1
    for (int bk = 0; bk < kChunk / 16; ++bk) {
      float xb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) xb[i] = (16 * bk + i == j) ? 1.f : 0.f;
#pragma unroll 1
      for (int c4 = 0; c4 < 4 * bk; ++c4) {   // columns s = 4 c4 .. 4 c4 + 3 of the earlier blocks
        const float x0 = X[(4 * c4 + 0) * kChunk + j], x1 = X[(4 * c4 + 1) * kChunk + j];
        const float x2 = X[(4 * c4 + 2) * kChunk + j], x3 = X[(4 * c4 + 3) * kChunk + j];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 a4 = *reinterpret_cast<const float4*>(A + (16 * bk + i) * AP + 4 * c4);
          xb[i] = fmaf(-a4.x, x0, xb[i]);
          xb[i] = fmaf(-a4.y, x1, xb[i]);
          xb[i] = fmaf(-a4.z, x2, xb[i]);
          xb[i] = fmaf(-a4.w, x3, xb[i]);
        }
      }
      const float* Ad = A + (16 * bk) * AP + 16 * bk;
#pragma unroll
      for (int i = 1; i < 16; ++i)
#pragma unroll
        for (int s2 = 0; s2 < i; ++s2) xb[i] = fmaf(-Ad[i * AP + s2], xb[s2], xb[i]);
#pragma unroll
      for (int i = 0; i < 16; ++i) X[(16 * bk + i) * kChunk + j] = xb[i];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < kChunk * 8; idx += 128) {   // T image (row r, K = column) from X
    const int r = idx >> 3, c = idx & 7;
    uint4 hv, lv;
    split8_bf16(X + r * kChunk + 8 * c, hv, lv);
    const uint32_t off = static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4);
    *reinterpret_cast<uint4*>(TI + off) = hv;
    *reinterpret_cast<uint4*>(TI + 8192 + off) = lv;
  }
  __syncthreads();   // X is consumed: the V and K images take its place
  {   // the diag(b) V and diag(b gamma) K images (row = feature, K = token): thread = feature row
    const int f = tid;
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      const bool isk = part == 1;
      uint8_t* dst = isk ? KI : VI;
      const float* scale = isk ? bgm : bb;
      const bool rowlive = f < DK;
      float v[kChunk];   // the whole row in flight at once
#pragma unroll
      for (int r = 0; r < kChunk; ++r)
        v[r] = (rowlive && r < n) ? b.y[static_cast<long long>(t0 + r) * b.ldy + (isk ? ko : vo) + f] : 0.f;
#pragma unroll
      for (int r = 0; r < kChunk; ++r) v[r] *= scale[r];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 hv, lv;
        split8_bf16(v + 8 * c, hv, lv);
        const uint32_t off = static_cast<uint32_t>(f) * 128u + ((static_cast<uint32_t>(c) ^ (f & 7u)) << 4);
        *reinterpret_cast<uint4*>(dst + off) = hv;
        *reinterpret_cast<uint4*>(dst + 16384 + off) = lv;
      }
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // ---- (3) D_U = (diag(b) V)^T T^T (columns 64..127), D_W = (diag(b gamma) K)^T T^T (128..191)
  if (tid == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(128, 64);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t th = tc::desc_kmajor_sw128(TI + kk * 32), tl = tc::desc_kmajor_sw128(TI + 8192 + kk * 32);
      const uint64_t vh = tc::desc_kmajor_sw128(VI + kk * 32), vl = tc::desc_kmajor_sw128(VI + 16384 + kk * 32);
      const uint64_t kh = tc::desc_kmajor_sw128(KI + kk * 32), kl = tc::desc_kmajor_sw128(KI + 16384 + kk * 32);
      tc::mma_bf16(tbase + 64, vh, th, idesc, kk ? 1u : 0u);
      tc::mma_bf16(tbase + 64, vh, tl, idesc, 1u);
      tc::mma_bf16(tbase + 64, vl, th, idesc, 1u);
      tc::mma_bf16(tbase + 128, kh, th, idesc, kk ? 1u : 0u);
      tc::mma_bf16(tbase + 128, kh, tl, idesc, 1u);
      tc::mma_bf16(tbase + 128, kl, th, idesc, 1u);
    }
    tc::mma_commit(bar);
  }
  if (!mbar_wait(bar, 1, abort, kWyWaitNs)) {
    if (!*abort) atomicOr(b.err, MK_DEVERR_PIPE_TIMEOUT);
    *abort = 1;
  }
  tc::fence_after_sync();
  // ---- epilogue: lane i holds U[r][i] and W[r][i] over the chunk's r
  if (!*abort) {
    const int f = tid;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float d[16];
      tc::tmem_ld16(tbase + lane_off + 64 + 16 * q, d);
      if (f < DV) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int r = 16 * q + u;
          if (r < n) b.u[static_cast<long long>(t0 + r) * Hd * DV + h * DV + f] = d[u];
        }
      }
    }
    // W rows (rows 64 + r of A1, K = feature; rows past the prompt zero): staged as the
    // image's 64 rows in shared memory (the V / K images are consumed), then copied out in
    // 16-byte pieces
    uint8_t* ws = sm + Lyt::kImg;   // [hi: KB blocks][lo: KB blocks] of 64 rows x 128 B
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float d[16];
      tc::tmem_ld16(tbase + lane_off + 128 + 16 * q, d);
      if (f < DK) {
        const int kb = f >> 6, kf = f & 63;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int r = 16 * q + u;
          put_bf16_pair(ws + kb * 8192, KB * 8192, r, kf, r < n ? d[u] : 0.f);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 256);
  if (*abort) return;
  {   // row r of the staged tile is row 64 + r of A1: the same swizzle phase (64 = 0 mod 8)
    const uint8_t* ws = sm + Lyt::kImg;
    for (int idx = tid; idx < 2 * KB * 64 * 8; idx += 128) {
      const int blk = idx >> 9, rem = idx & 511;   // blk: part * KB + kb; rem: row * 8 + chunk
      *reinterpret_cast<uint4*>(a1 + blk * 16384 + 64 * 128 + rem * 16) =
          *reinterpret_cast<const uint4*>(ws + blk * 8192 + rem * 16);
    }
  }
}


template <int DK>
constexpr size_t wy_tc_smem() {
  return WyImg<DK>::kA1 + 2ull * (WyImg<DK>::kP + WyImg<DK>::kKT) + 2ull * (DK / 64) * 2048 + 2 * 4096 +
         sizeof(float) * (2 * kChunk * kRowGroup + 2 * kChunk + 128) + sizeof(WyTcBars) + 1024;
}

template <int DK, int DV>
__global__ void __launch_bounds__(128, 1) wy_state_tc(WyBufs b, float* __restrict__ S) {
  using I = WyImg<DK>;
  constexpr int KB = DK / 64, RG = kRowGroup;
  constexpr uint32_t kPK = I::kP + I::kKT, kB1 = 2u * KB * 2048u;
  constexpr uint32_t idesc = tc::idesc_bf16_f32(128, 16);
  extern __shared__ uint8_t wy_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wy_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A1 = sm;
  uint8_t* PK0 = A1 + I::kA1;
  uint8_t* B1 = PK0 + 2 * kPK;
  uint8_t* B2 = B1 + kB1;
  uint8_t* B3 = B2 + 4096;
  float* Ub = reinterpret_cast<float*>(B3 + 4096);   // [2][64][16]
  float* dcb = Ub + 2 * kChunk * RG;                 // [2][64]
  float* gl = dcb + 2 * kChunk;                      // [128] gamma at each chunk's last row
  WyTcBars* bars = reinterpret_cast<WyTcBars*>(gl + 128);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int Hd = b.Hd, h = blockIdx.x, i0 = blockIdx.y * RG;
  const int nch = (b.T + kChunk - 1) / kChunk;
  auto img_at = [&](int c) { return b.img + (static_cast<size_t>(c) * Hd + h) * I::kBytes; };
  volatile int* abort = &bars->abort;

  if (tid == 0) {
    mbar_init(&bars->a1, 1);
    mbar_init(&bars->pk[0], 1);
    mbar_init(&bars->pk[1], 1);
    mbar_init(&bars->mma, 1);
    mbar_init(&bars->mmas, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&bars->tmem, 64);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
  // D1 of chunk c in columns 16 (c & 1) .. + 15 (o of chunk c is read during chunk c + 1),
  // D3 (S^T) in columns 32 .. 47
  auto d1_of = [&](int c) { return bars->tmem + 16u * static_cast<uint32_t>(c & 1) + lane_off; };
  const uint32_t d3 = bars->tmem + 32 + lane_off;

  int n_a1 = 0, n_pk[2] = {0, 0};   // bulk copies issued per barrier (thread 0)
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars->a1, I::kA1);
    tc::bulk_load(A1, img_at(0), I::kA1, &bars->a1);
    n_a1 = 1;
    for (int c = 0; c < 2 && c < nch; ++c) {
      mbar_arrive_expect_tx(&bars->pk[c], kPK);
      tc::bulk_load(PK0 + c * kPK, img_at(c) + I::kA1, kPK, &bars->pk[c]);
      n_pk[c] = 1;
    }
  }
  auto fetch_ud = [&](int c) {   // U columns i0.., decay of chunk c (rows past the prompt read as zero)
    const int t0 = c * kChunk, n = min(kChunk, b.T - t0);
    float* U = Ub + (c & 1) * kChunk * RG;
    for (int idx = tid; idx < kChunk * RG / 4; idx += 128) {
      const int r = idx >> 2, q4 = idx & 3;
      const long long t = t0 + min(r, n - 1);
      cp_async16(U + r * RG + 4 * q4, b.u + t * Hd * DV + h * DV + i0 + 4 * q4, r < n ? 16u : 0u);
    }
    if (tid < kChunk) {
      const long long t = t0 + min(tid, n - 1);
      cp_async4(dcb + (c & 1) * kChunk + tid, b.dec + t * Hd + h, tid < n ? 4u : 0u);
    }
  };
  fetch_ud(0);
  cp_async_commit();
  for (int c = tid; c < nch; c += 128) {
    const int tl = min(b.T, (c + 1) * kChunk) - 1;
    gl[c] = b.gam[static_cast<long long>(tl) * Hd + h];
  }
  // S0 operand tile (rows i of S, K = dk) from thread j = column j, bf16 high and low parts
  auto put_s = [&](const float* sv) {
    if (tid < DK) {
      const int kb = tid >> 6, kk = tid & 63;
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const uint16_t hi = f_to_bf16(sv[i]), lo = f_to_bf16(sv[i] - bf16_to_f(hi));
        const uint32_t off = tc::sw128_offset(i, kk);
        *reinterpret_cast<uint16_t*>(B1 + kb * 2048 + off) = hi;
        *reinterpret_cast<uint16_t*>(B1 + (KB + kb) * 2048 + off) = lo;
      }
    }
  };
  // o of chunk c (lanes 0..63 of its D1) to global; warps 0 and 1, every lane takes part
  auto store_o = [&](int c) {
    const int t0 = c * kChunk, n = min(kChunk, b.T - t0);
    float o[RG];
    tc::tmem_ld16(d1_of(c), o);
    if (tid < n) {
      float4* dst = reinterpret_cast<float4*>(b.o + static_cast<long long>(t0 + tid) * Hd * DV + h * DV + i0);
#pragma unroll
      for (int q = 0; q < RG / 4; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
  };
  float sv[RG];
#pragma unroll
  for (int i = 0; i < RG; ++i)
    sv[i] = tid < DK ? S[(static_cast<long long>(h) * DV + i0 + i) * DK + tid] : 0.f;
  __syncthreads();   // gl
  put_s(sv);
  {
    float v[RG];
#pragma unroll
    for (int i = 0; i < RG; ++i) v[i] = gl[0] * sv[i];
    tc::tmem_st16(d3, v);
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  uint32_t mph = 0, sph = 0;
  for (int ch = 0; ch < nch; ++ch) {
    // ---- A: D1(ch) = [gamma Q; W] S0^T
    if (tid == 0) {
      if (!mbar_wait(&bars->a1, ch & 1, abort, kWyWaitNs)) {
        if (!*abort) atomicOr(b.err, MK_DEVERR_PIPE_TIMEOUT);
        *abort = 1;
      } else {
        tc::fence_after_sync();
        const uint32_t d1 = d1_of(ch) - lane_off;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ah = tc::desc_kmajor_sw128(A1 + kb * 16384 + kk * 32);
            const uint64_t al = tc::desc_kmajor_sw128(A1 + (KB + kb) * 16384 + kk * 32);
            const uint64_t bh = tc::desc_kmajor_sw128(B1 + kb * 2048 + kk * 32);
            const uint64_t bl = tc::desc_kmajor_sw128(B1 + (KB + kb) * 2048 + kk * 32);
            tc::mma_bf16(d1, ah, bh, idesc, (kb | kk) ? 1u : 0u);
            tc::mma_bf16(d1, ah, bl, idesc, 1u);
            tc::mma_bf16(d1, al, bh, idesc, 1u);
          }
        tc::mma_commit(&bars->mma);
      }
    }
    // (MMAs complete in issue order: this wait also covers B of the previous chunk)
    if (!mbar_wait(&bars->mma, mph, abort, kWyWaitNs)) *abort = 1;
    mph ^= 1u;
    tc::fence_after_sync();
    if (tid == 0 && !*abort) {
      if (ch + 1 < nch) {   // A1 is consumed: stage the next chunk's
        mbar_arrive_expect_tx(&bars->a1, I::kA1);
        tc::bulk_load(A1, img_at(ch + 1), I::kA1, &bars->a1);
        ++n_a1;
      }
      if (ch >= 1 && ch + 1 < nch) {   // P / K^T of chunk ch - 1 are consumed: stage chunk ch + 1's
        const int bf = (ch + 1) & 1;
        mbar_arrive_expect_tx(&bars->pk[bf], kPK);
        tc::bulk_load(PK0 + bf * kPK, img_at(ch + 1) + I::kA1, kPK, &bars->pk[bf]);
        ++n_pk[bf];
      }
    }
    if (ch + 1 < nch) fetch_ud(ch + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();   // U and the decay factors of this chunk
    if (*abort) break;
    if (warp < 2) {
      if (ch > 0) store_o(ch - 1);   // o of the previous chunk, off the state's critical path
    } else {
      // ---- Delta = U - W S0^T; the tiles Delta^T and (dec Delta)^T (row i, K = token r)
      const int r = tid - 64;
      float ws[RG];
      tc::tmem_ld16(d1_of(ch), ws);
      const float* U = Ub + (ch & 1) * kChunk * RG;
      const float dr = dcb[(ch & 1) * kChunk + r];
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const float d = U[r * RG + i] - ws[i];
        const float dd = dr * d;
        const uint32_t off = tc::sw128_offset(i, r);
        const uint16_t h1 = f_to_bf16(d), h2 = f_to_bf16(dd);
        *reinterpret_cast<uint16_t*>(B2 + off) = h1;
        *reinterpret_cast<uint16_t*>(B2 + 2048 + off) = f_to_bf16(d - bf16_to_f(h1));
        *reinterpret_cast<uint16_t*>(B3 + off) = h2;
        *reinterpret_cast<uint16_t*>(B3 + 2048 + off) = f_to_bf16(dd - bf16_to_f(h2));
      }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    // ---- C: D3 += K^T (dec Delta) (the state: committed on its own), then B: D1(ch)[0..63] += P Delta
    if (tid == 0) {
      if (!mbar_wait(&bars->pk[ch & 1], (ch >> 1) & 1, abort, kWyWaitNs)) {
        if (!*abort) atomicOr(b.err, MK_DEVERR_PIPE_TIMEOUT);
        *abort = 1;
      } else {
        tc::fence_after_sync();
        const uint8_t* PK = PK0 + (ch & 1) * kPK;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t kh = tc::desc_kmajor_sw128(PK + I::kP + kk * 32);
          const uint64_t kl = tc::desc_kmajor_sw128(PK + I::kP + 16384 + kk * 32);
          const uint64_t eh = tc::desc_kmajor_sw128(B3 + kk * 32);
          const uint64_t el = tc::desc_kmajor_sw128(B3 + 2048 + kk * 32);
          tc::mma_bf16(d3 - lane_off, kh, eh, idesc, 1u);
          tc::mma_bf16(d3 - lane_off, kh, el, idesc, 1u);
          tc::mma_bf16(d3 - lane_off, kl, eh, idesc, 1u);
        }
        tc::mma_commit(&bars->mmas);
        const uint32_t d1 = d1_of(ch) - lane_off;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ph = tc::desc_kmajor_sw128(PK + kk * 32);
          const uint64_t pl = tc::desc_kmajor_sw128(PK + 8192 + kk * 32);
          const uint64_t dh = tc::desc_kmajor_sw128(B2 + kk * 32);
          const uint64_t dl = tc::desc_kmajor_sw128(B2 + 2048 + kk * 32);
          tc::mma_bf16(d1, ph, dh, idesc, 1u);
          tc::mma_bf16(d1, ph, dl, idesc, 1u);
          tc::mma_bf16(d1, pl, dh, idesc, 1u);
        }
      }
    }
    if (!mbar_wait(&bars->mmas, sph, abort, kWyWaitNs)) *abort = 1;
    sph ^= 1u;
    tc::fence_after_sync();
    if (*abort) break;
    // ---- the state after this chunk
    tc::tmem_ld16(d3, sv);
    if (ch + 1 < nch) {
      put_s(sv);
      float v[RG];
#pragma unroll
      for (int i = 0; i < RG; ++i) v[i] = gl[ch + 1] * sv[i];
      tc::tmem_st16(d3, v);
    } else if (tid < DK) {
#pragma unroll
      for (int i = 0; i < RG; ++i) S[(static_cast<long long>(h) * DV + i0 + i) * DK + tid] = sv[i];
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  // o of the last chunk once its B has completed
  if (!*abort && nch > 0) {
    if (tid == 0) tc::mma_commit(&bars->mma);
    if (!mbar_wait(&bars->mma, mph, abort, kWyWaitNs)) *abort = 1;
    tc::fence_after_sync();
    if (!*abort && warp < 2) store_o(nch - 1);
  }
  cp_async_wait<0>();
  if (tid == 0) {   // let issued bulk copies land before the CTA ends (bounded)
    int never = 0;
    if (n_a1 > 0) mbar_wait(&bars->a1, (n_a1 - 1) & 1, &never, kWyWaitNs / 5);
    for (int c = 0; c < 2; ++c)
      if (n_pk[c] > 0) mbar_wait(&bars->pk[c], (n_pk[c] - 1) & 1, &never, kWyWaitNs / 5);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(bars->tmem, 64);
}

template <int DK, int DV>
size_t wy_fast_smem(bool state_pass) {
  const size_t prep = sizeof(float) * (2 * kChunk * (DK + 4) + kChunk * (kChunk + 4) + 2 * kChunk);
  const size_t state = sizeof(float) * (kRowGroup * (DK + 4) + 3 * kChunk * (DK + 4) + kChunk * (kChunk + 4) +
                                        kRowGroup * (kChunk + 4) + kChunk * kRowGroup + 4 * kChunk);
  return state_pass ? state : prep;
}

size_t wy_prep_smem(int dk, int dv) {
  return sizeof(float) * (2 * kChunk * (dk + 1) + kChunk * (dv + dk) + kChunk * 65 + 2 * kChunk);
}
size_t wy_state_smem(int dk) {
  return sizeof(float) * (kRowGroup * (dk + 1) + 2 * kChunk * (dk + 1) + kChunk * dk + kChunk * 65 +
                          kChunk * kRowGroup + kChunk * 17 + 2 * kChunk);
}

// ------------------------------------------------------------------ attention as two GEMMs
// For long prompts, per query head: S = Q K^T (tcgen05 linear layer over the cached keys),
// P = causal softmax(S) written as bf16 high/low parts, O = P V (second linear layer
// against V^T). Keys past a row's position are masked in the softmax; P is zero there.
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < static_cast<int>(blockDim.x >> 5)) ? red[l] : -INFINITY;
  return warp_max(t);
}

// VT[d][j] = V[j][d] for the keys up to the pass's last position, zero past it.
__global__ void v_transpose(const uint16_t* __restrict__ vg, int D, int nk, const int* __restrict__ posp, int last_off,
                            int max_ctx, uint16_t* __restrict__ vt) {
  __shared__ uint16_t tile[32][33];
  const int last = min(*posp + last_off, max_ctx - 1);
  const int j0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int j = j0 + k, d = d0 + threadIdx.x;
    tile[k][threadIdx.x] = (j <= last && d < D) ? vg[static_cast<long long>(j) * D + d] : 0;
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int d = d0 + k, j = j0 + threadIdx.x;
    if (d < D && j < nk) vt[static_cast<long long>(d) * nk + j] = tile[threadIdx.x][k];
  }
}

// ------------------------------------------------------------------ causal attention
// One CTA per (query token t, kv head g): the Hq/Hkv query heads of group g attend to the
// cached positions 0 .. pos0+t in blocks of 64 keys with an online softmax.
constexpr int kKeyBlock = 64;
constexpr int kMaxDraftRows = 17;   // max_draft <= 16
constexpr int kFlashAttnMinRows = 64;   // prompts from this many tokens run the flash attention

// With nsplit > 1 (few tokens: T * Hkv CTAs would leave most SMs idle) CTA z takes the
// z-th of nsplit equal ranges of the token's keys and writes its unnormalised partial
// (acc[D], m, l per query head) to part [T][Hq][nsplit][D + 2]; attn_combine merges them.
__global__ void __launch_bounds__(256) attn_prefill(const float* __restrict__ q, int ldq, const uint16_t* __restrict__ kc,
                                                    const uint16_t* __restrict__ vc, const int* __restrict__ posp,
                                                    int off, int Hq, int Hkv, int D, int max_ctx, float* __restrict__ o,
                                                    int ldo, int nsplit, float* __restrict__ part) {
  extern __shared__ float sm[];
  const int t = blockIdx.x, g = blockIdx.y, grp = Hq / Hkv, z = blockIdx.z;
  const int nall = min(*posp + off + t + 1, max_ctx);
  const int ks = ((nall + nsplit - 1) / nsplit + kKeyBlock - 1) / kKeyBlock * kKeyBlock;
  const int kbeg = min(nall, z * ks), nkeys = min(nall, kbeg + ks);
  float* qs = sm;                                   // [grp][D]
  float* sc = qs + grp * D;                         // [grp][64]
  float* ml = sc + grp * kKeyBlock;                 // [grp][3]: m, l, corr
  uint16_t* kb = reinterpret_cast<uint16_t*>(ml + 3 * 8);   // [64][D]
  uint16_t* vb = kb + kKeyBlock * D;                // [64][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int idx = threadIdx.x; idx < grp * D; idx += blockDim.x)
    qs[idx] = q[static_cast<long long>(t) * ldq + (g * grp) * D + idx];
  if (threadIdx.x < grp) {
    ml[3 * threadIdx.x] = -INFINITY;
    ml[3 * threadIdx.x + 1] = 0.f;
    ml[3 * threadIdx.x + 2] = 0.f;
  }
  float acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u] = 0.f;
  const uint16_t* kg = kc + static_cast<long long>(g) * max_ctx * D;
  const uint16_t* vg = vc + static_cast<long long>(g) * max_ctx * D;
  for (int p0 = kbeg; p0 < nkeys; p0 += kKeyBlock) {
    const int np = min(kKeyBlock, nkeys - p0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < np * D / 8; idx += blockDim.x) {
      reinterpret_cast<uint4*>(kb)[idx] = reinterpret_cast<const uint4*>(kg + static_cast<long long>(p0) * D)[idx];
      reinterpret_cast<uint4*>(vb)[idx] = reinterpret_cast<const uint4*>(vg + static_cast<long long>(p0) * D)[idx];
    }
    __syncthreads();
    for (int pp = warp; pp < np; pp += 8) {        // scores: warp per key, lanes over D
      float d[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) d[u] = 0.f;
      for (int i = lane; i < D; i += 32) {
        const float kv = bf16_to_f(kb[pp * D + i]);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (u < grp) d[u] = fmaf(qs[u * D + i], kv, d[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < grp) {
          d[u] = warp_sum(d[u]);
          if (lane == 0) sc[u * kKeyBlock + pp] = d[u];
        }
    }
    __syncthreads();
    if (warp < grp) {                               // online softmax, warp per query head
      float mx = -INFINITY;
      for (int pp = lane; pp < np; pp += 32) mx = fmaxf(mx, sc[warp * kKeyBlock + pp]);
      mx = warp_max(mx);
      const float m_old = ml[3 * warp], m_new = fmaxf(m_old, mx);
      float ls = 0.f;
      for (int pp = lane; pp < np; pp += 32) {
        const float e = expf(sc[warp * kKeyBlock + pp] - m_new);
        sc[warp * kKeyBlock + pp] = e;
        ls += e;
      }
      ls = warp_sum(ls);
      __syncwarp();
      if (lane == 0) {
        const float corr = expf(m_old - m_new);
        ml[3 * warp] = m_new;
        ml[3 * warp + 1] = ml[3 * warp + 1] * corr + ls;
        ml[3 * warp + 2] = corr;
      }
    }
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += blockDim.x) {   // values: thread per dim (D <= 256)
      float vs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vs[u] = 0.f;
      for (int pp = 0; pp < np; ++pp) {
        const float vv = bf16_to_f(vb[pp * D + d]);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (u < grp) vs[u] = fmaf(sc[u * kKeyBlock + pp], vv, vs[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < grp) acc[u] = acc[u] * ml[3 * u + 2] + vs[u];
    }
  }
  __syncthreads();
  if (nsplit > 1) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < grp) part[((static_cast<long long>(t) * Hq + g * grp + u) * nsplit + z) * (D + 2) + d] = acc[u];
    }
    if (threadIdx.x < grp) {
      float* pp = part + ((static_cast<long long>(t) * Hq + g * grp + threadIdx.x) * nsplit + z) * (D + 2);
      pp[D] = ml[3 * threadIdx.x];
      pp[D + 1] = ml[3 * threadIdx.x + 1];
    }
    return;
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u < grp) o[static_cast<long long>(t) * ldo + (g * grp + u) * D + d] = acc[u] / ml[3 * u + 1];
  }
}

// o[t][hq] = sum_z e^{m_z - M} acc_z / sum_z e^{m_z - M} l_z over the key splits (empty
// splits carry m = -inf, l = 0).
__global__ void attn_combine(const float* __restrict__ part, int nsplit, int Hq, int D, float* __restrict__ o, int ldo) {
  const int t = blockIdx.x, hq = blockIdx.y;
  const float* pp = part + (static_cast<long long>(t) * Hq + hq) * nsplit * (D + 2);
  float M = -INFINITY;
  for (int z = 0; z < nsplit; ++z) M = fmaxf(M, pp[z * (D + 2) + D]);
  float L = 0.f;
  for (int z = 0; z < nsplit; ++z) {
    const float mz = pp[z * (D + 2) + D];
    if (mz > -INFINITY) L += expf(mz - M) * pp[z * (D + 2) + D + 1];
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int z = 0; z < nsplit; ++z) {
      const float mz = pp[z * (D + 2) + D];
      if (mz > -INFINITY) acc = fmaf(expf(mz - M), pp[z * (D + 2) + d], acc);
    }
    o[static_cast<long long>(t) * ldo + hq * D + d] = acc / L;
  }
}

size_t attn_prefill_smem(int grp, int D) {
  return sizeof(float) * (grp * D + grp * kKeyBlock + 3 * 8) + 2 * sizeof(uint16_t) * kKeyBlock * D;
}

}  // namespace
}  // namespace mk

namespace mk {
namespace {

__global__ void check_capacity(const int* pos, int n, int max_ctx, int* err) {
  if (*pos + n > max_ctx) atomicOr(err, MK_DEVERR_CAPACITY);
}
__global__ void advance_pos(int* pos, int n, int max_ctx) {
  *pos = min(*pos + n, max_ctx);
}

// Greedy token of each logits row (lowest index among equal maxima): CTA (t, c) scans
// slice c of row t and folds its best packed (value, index) key into best[t] (zeroed
// before); the maximum is the same in any order.
__global__ void row_argmax(const float* __restrict__ logits, int V, unsigned long long* __restrict__ best) {
  __shared__ unsigned long long wb[32];
  const float* r = logits + static_cast<long long>(blockIdx.x) * V;
  const int per = (V + gridDim.y - 1) / gridDim.y;
  const int i0 = blockIdx.y * per, i1 = min(V, i0 + per);
  unsigned long long b = 0;
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const unsigned long long k = pack_argmax(r[i], i);
    b = k > b ? k : b;
  }
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long x = __shfl_xor_sync(0xffffffffu, b, o);
    b = x > b ? x : b;
  }
  if ((threadIdx.x & 31) == 0) wb[threadIdx.x >> 5] = b;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = wb[w] > b ? wb[w] : b;
    atomicMax(best + blockIdx.x, b);
  }
}

// Commit of a verify pass to its accepted prefix: tokens 0 .. n of the pass (n = *n_acc)
// enter the state, S = e^{g_n} S0 + sum_{r<=n} e^{g_n - g_r} Delta_r k_r^T, for one row
// group of one head.
__global__ void __launch_bounds__(256) commit_state(float* __restrict__ S, const float* __restrict__ delta,
                                                    const float* __restrict__ kk, const float* __restrict__ g,
                                                    const int* __restrict__ n_acc, int Hd, int dk, int dv) {
  const int h = blockIdx.x, i0 = blockIdx.y * kRowGroup;
  const int last = *n_acc;
  const float gl = g[static_cast<long long>(last) * Hd + h];
  for (int idx = threadIdx.x; idx < kRowGroup * dk; idx += blockDim.x) {
    const int i = i0 + idx / dk, j = idx % dk;
    float* sp = S + (static_cast<long long>(h) * dv + i) * dk + j;
    float acc = expf(gl) * *sp;
    for (int r = 0; r <= last; ++r)
      acc = fmaf(expf(gl - g[static_cast<long long>(r) * Hd + h]) * delta[static_cast<long long>(r) * Hd * dv + h * dv + i],
                 kk[static_cast<long long>(r) * Hd * dk + h * dk + j], acc);
    *sp = acc;
  }
}

// Conv history of the accepted prefix: the raw inputs of its last W-1 tokens.
__global__ void commit_conv(const float* __restrict__ raw, float* __restrict__ ring, int W, int C,
                            const int* __restrict__ posp, const int* __restrict__ n_acc) {
  const int m = blockIdx.y, r = *n_acc - m;
  if (r < 0) return;
  const int p = *posp + r;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < C; c += gridDim.x * blockDim.x)
    ring[static_cast<long long>(p % W) * C + c] = raw[static_cast<long long>(r) * C + c];
}

// The greedy token of a row_argmax result (lowest index among equal maxima).
__global__ void argmax_token(const unsigned long long* best, int32_t* out) {
  *out = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(*best & 0xFFFFFFFFull));
}

__global__ void advance_pos_accepted(int* pos, const int* n_acc, int max_ctx) {
  *pos = min(*pos + *n_acc + 1, max_ctx);
}

__global__ void accept_prefix(const int* tokens, const unsigned long long* best, int K, int* n_out, int* n_acc, int* out,
                              int* greedy) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int g[kMaxDraftRows];
  for (int i = 0; i <= K; ++i) {
    g[i] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best[i] & 0xFFFFFFFFull));
    greedy[i] = g[i];
  }
  int n = 0;
  while (n < K && tokens[1 + n] == g[n]) ++n;
  for (int i = 0; i < n; ++i) out[i] = tokens[1 + i];
  out[n] = g[n];
  *n_out = n;
  *n_acc = n;
}

// ---------------------------------------------------------------- sampled acceptance
// Sampling-mode speculative verify. The open-jet Qwen3.8-27B megakernel follow-up (speed
// section) states that with sampling, speculation keeps the distribution the model has
// without drafts; the rule is standard speculative sampling (Leviathan et al. 2023, Chen et
// al. 2023) with each draft a point mass: draft d at position i is kept iff u[2i] < p_i(d),
// p_i = softmax(z_i / tau); at the first rejection the output token is drawn from p_i with d
// removed, else after K kept drafts from p_K, by the inverse of the cumulative distribution
// with u[2i + 1] (the smallest token index whose running weight exceeds u * total).
// The weights, sums and thresholds are float64: with V ~ 1.5e5 tokens the cumulative
// boundaries lie ~1e-5 apart, well inside float32's summation error, and the decision
// should depend on the logits and the uniforms only.

// Weight of a token relative to its row's maximum m; the maximum itself weighs exactly 1.
__device__ __forceinline__ double samp_weight(float z, double m, double inv_tau) {
  return exp((static_cast<double>(z) - m) * inv_tau);
}

template <bool kMax, typename F>
__device__ __forceinline__ F block_reduce(F v, F* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) {
    const F x = __shfl_xor_sync(0xffffffffu, v, o);
    v = kMax ? (x > v ? x : v) : v + x;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : (kMax ? static_cast<F>(-INFINITY) : F(0));
    for (int o = 16; o > 0; o >>= 1) {
      const F x = __shfl_xor_sync(0xffffffffu, v, o);
      v = kMax ? (x > v ? x : v) : v + x;
    }
    if (lane == 0) red[32] = v;
  }
  __syncthreads();
  v = red[32];
  __syncthreads();
  return v;
}

constexpr int kSampThreads = 256;

// Slice sl of logits row t (kSampSlices slices per row): part[(t * kSampSlices + sl) * 2] = the
// slice maximum m_s, [+1] = sum of exp((z - m_s) / tau) over the slice (an empty slice: -inf, 0).
__global__ void __launch_bounds__(kSampThreads) row_softmax_partials(const float* __restrict__ logits, int V,
                                                                     double inv_tau, double* __restrict__ part) {
  __shared__ float redf[33];
  __shared__ double redd[33];
  const int t = blockIdx.x, sl = blockIdx.y;
  const int L = (V + kSampSlices - 1) / kSampSlices;
  const int j0 = sl * L, j1 = min(V, j0 + L);
  const float* r = logits + static_cast<long long>(t) * V;
  float mf = -INFINITY;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) mf = fmaxf(mf, r[j]);
  const double m = block_reduce<true>(mf, redf);
  double s = 0.0;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) s += samp_weight(r[j], m, inv_tau);
  s = block_reduce<false>(s, redd);
  if (threadIdx.x == 0) {
    part[(t * kSampSlices + sl) * 2] = m;
    part[(t * kSampSlices + sl) * 2 + 1] = s;
  }
}

// One warp: row statistics (maximum M, Z = sum over slices of sum_s exp((m_s - M) / tau)) and
// the draft tests in order. Every lane computes the same values (the butterfly sums are
// order-symmetric), so the loop runs in lockstep; lane 0 writes the decision.
__global__ void samp_decide(const int* __restrict__ tokens, int K, const float* __restrict__ logits, int V,
                            double inv_tau, const double* __restrict__ part, const float* __restrict__ uni,
                            SampDecision* __restrict__ dec) {
  const int lane = threadIdx.x;
  int n = 0;
  double M = 0.0;
  for (;;) {
    double ms = -INFINITY, ss = 0.0;
    if (lane < kSampSlices) {
      ms = part[(n * kSampSlices + lane) * 2];
      ss = part[(n * kSampSlices + lane) * 2 + 1];
    }
    double mx = ms;
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double z = ss > 0.0 ? ss * exp((ms - mx) * inv_tau) : 0.0;
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    M = mx;
    if (n >= K) break;
    const int d = tokens[1 + n];
    double pd = 0.0;
    if (d >= 0 && d < V) pd = samp_weight(logits[static_cast<long long>(n) * V + d], M, inv_tau) / z;
    if (static_cast<double>(uni[2 * n]) < pd) ++n;
    else break;
  }
  if (lane == 0) {
    dec->M = M;
    dec->n = n;
    dec->excl = n < K ? tokens[1 + n] : -1;
  }
}

// Chunk c (kDrawChunks contiguous chunks) of the stopping row: the sum of its weights
// exp((z - M) / tau), the rejected draft left out.
__global__ void __launch_bounds__(kSampThreads) samp_chunk_sums(const float* __restrict__ logits, int V,
                                                                double inv_tau, const SampDecision* __restrict__ dec,
                                                                double* __restrict__ csum) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= kDrawChunks) return;
  const int n = dec->n, excl = dec->excl;
  const double M = dec->M;
  const float* r = logits + static_cast<long long>(n) * V;
  const int per = (V + kDrawChunks - 1) / kDrawChunks;
  const int j0 = c * per, j1 = min(V, j0 + per);
  double s = 0.0;
  for (int j = j0; j < j1; ++j)
    if (j != excl) s += samp_weight(r[j], M, inv_tau);
  csum[c] = s;
}

// One warp: the draw by the inverse CDF, walked in index order at three levels (groups of
// kDrawGroup chunks, chunks, tokens). Each level's running sum adds the same terms in the
// same order as the sum it is compared with, so it only grows and its last value equals that
// sum; rounding between levels is caught by taking the last token with weight.
__global__ void samp_select(const int* __restrict__ tokens, const float* __restrict__ logits, int V, double inv_tau,
                            const SampDecision* __restrict__ dec, const double* __restrict__ csum,
                            const float* __restrict__ uni, int* n_out, int* n_acc, int* out) {
  constexpr int kGroups = kDrawChunks / kDrawGroup;
  __shared__ double gsum[kGroups];
  const int lane = threadIdx.x;
  for (int g = lane; g < kGroups; g += 32) {
    double s = 0.0;
    for (int i = 0; i < kDrawGroup; ++i) s += csum[g * kDrawGroup + i];
    gsum[g] = s;
  }
  __syncwarp();
  if (lane != 0) return;
  const int n = dec->n, excl = dec->excl;
  const double M = dec->M;
  double total = 0.0;
  int last_g = -1;
  for (int g = 0; g < kGroups; ++g) {
    total += gsum[g];
    if (gsum[g] > 0.0) last_g = g;
  }
  const double target = static_cast<double>(uni[2 * n + 1]) * total;
  int g = -1;
  double before = 0.0, run = 0.0;
  for (int i = 0; i < kGroups; ++i) {
    const double nxt = run + gsum[i];
    if (nxt > target) {
      g = i;
      before = run;
      break;
    }
    run = nxt;
  }
  if (g < 0 && last_g >= 0) {   // u * total rounded up to total
    g = last_g;
    before = 0.0;
    for (int i = 0; i < g; ++i) before += gsum[i];
  }
  int tok = excl;               // no other token has weight (only if u[2n] >= 1)
  if (g >= 0) {
    const double* cs = csum + g * kDrawGroup;
    const double rem = target - before;
    int c = -1, last_c = -1;
    double before2 = 0.0, run2 = 0.0;
    for (int i = 0; i < kDrawGroup; ++i) {
      if (cs[i] > 0.0) last_c = i;
      const double nxt = run2 + cs[i];
      if (c < 0 && nxt > rem) {
        c = i;
        before2 = run2;
      }
      run2 = nxt;
    }
    if (c < 0) {
      c = last_c;
      before2 = 0.0;
      for (int i = 0; i < c; ++i) before2 += cs[i];
    }
    if (c < 0) c = 0;             // not reached: a group with weight has a chunk with weight
    const double rem2 = rem - before2;
    const float* r = logits + static_cast<long long>(n) * V;
    const int per = (V + kDrawChunks - 1) / kDrawChunks;
    const int j0 = (g * kDrawGroup + c) * per, j1 = min(V, j0 + per);
    double acc = 0.0;
    int lastpos = -1;
    tok = -1;
    for (int j = j0; j < j1; ++j) {
      if (j == excl) continue;
      const double w = samp_weight(r[j], M, inv_tau);
      if (w > 0.0) lastpos = j;
      acc += w;
      if (acc > rem2) {
        tok = j;
        break;
      }
    }
    if (tok < 0) tok = lastpos;
  }
  for (int i = 0; i < n; ++i) out[i] = tokens[1 + i];
  out[n] = tok;
  *n_out = n;
  *n_acc = n;
}

// One pass of every layer over T tokens at device position *pos + off. With vs (a verify
// pass, T <= 64) the DeltaNet layers keep their state and conv history untouched and
// save what the commit of an accepted prefix needs.
// Row bytes of a 4-bit matrix with K inputs (K a multiple of 256).
inline long long q4_row_bytes(long long K) { return (K / 256) * 144; }

// 4-bit linear layer over the T tokens' bf16 high / low activation parts [T][K].
cudaError_t launch_q4_linear(const uint16_t* xhi, const uint16_t* xlo, const void* W, long long ldw, float* C,
                             long long ldc, int T, int N, int K, int accumulate, float* ws, long long ws_floats,
                             cudaStream_t s) {
  if (T <= 0 || N <= 0) return cudaSuccess;
  const int tiles = (N + 127) / 128, ttiles = (T + 7) / 8, nsb = K / 256;
  int nz = std::min(nsb, std::max(1, (4 * 148 + tiles * ttiles - 1) / (tiles * ttiles)));
  if (static_cast<long long>(nz) * T * N > ws_floats) nz = 1;
  int per = (nsb + nz - 1) / nz;
  nz = (nsb + per - 1) / per;
  if (nz <= 1) per = nsb;
  constexpr size_t smem = 4ull * kQ4Depth * 32 * 144;
  q4_linear_mma<<<dim3(tiles, nz, ttiles), 128, smem, s>>>(xhi, xlo, K, static_cast<const uint8_t*>(W), ldw,
                                                            nz > 1 ? ws : C, ldc, T, N, K, per, accumulate);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && nz > 1) {
    const long long tot = static_cast<long long>(T) * N;
    q4_split_reduce<<<static_cast<int>(std::min<long long>((tot + 255) / 256, 1184)), 256, 0, s>>>(ws, nz, T, N, C, ldc,
                                                                                               accumulate);
    e = cudaGetLastError();
  }
  return e;
}

// bf16 linear layer for few-token passes (T <= 8 per tile) over the tokens' bf16 high / low parts.
cudaError_t launch_bf16_linear(const uint16_t* xhi, const uint16_t* xlo, const void* W, long long ldw, float* C,
                               long long ldc, int T, int N, int K, int accumulate, float* ws, long long ws_floats,
                               cudaStream_t s) {
  if (T <= 0 || N <= 0) return cudaSuccess;
  const int tiles = (N + 127) / 128, ttiles = (T + 7) / 8, nkb = K / 64;
  int nz = std::min(nkb, std::max(1, (3 * 148 + tiles * ttiles - 1) / (tiles * ttiles)));
  if (static_cast<long long>(nz) * T * N > ws_floats) nz = 1;
  int per = (nkb + nz - 1) / nz;
  nz = (nkb + per - 1) / per;
  if (nz <= 1) per = nkb;
  constexpr size_t smem = 4ull * kBfDepth * 32 * 128;
  bf16_linear_mma<<<dim3(tiles, nz, ttiles), 128, smem, s>>>(xhi, xlo, K, static_cast<const uint8_t*>(W), ldw,
                                                              nz > 1 ? ws : C, ldc, T, N, K, per, accumulate);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && nz > 1) {
    const long long tot = static_cast<long long>(T) * N;
    q4_split_reduce<<<static_cast<int>(std::min<long long>((tot + 255) / 256, 1184)), 256, 0, s>>>(ws, nz, T, N, C, ldc,
                                                                                               accumulate);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t prefill_pass(mk_model* m, const int32_t* tok, int T, int off, cudaStream_t s,
                         const mk_verify_ws* vs = nullptr) {
  const mk_config& c = m->cfg;
  const DecodeParams& b = m->base;
  const mk_prefill_ws& pf = m->pf;
  const int H = c.hidden, F = c.ffn, C = b.C, Hd = c.dn_heads, dk = c.dn_dk, dv = c.dn_dv, Wc = c.conv_width;
  const int Hq = c.at_q_heads, Hkv = c.at_kv_heads, D = c.at_head_dim;
  const int qd = Hq * D;
  cudaError_t e = cudaSuccess;
  auto chk = [&]() {
    if (e == cudaSuccess) e = cudaGetLastError();
    ++m->launches;
  };
  const bool q4 = b.q4 != 0;   // 4-bit weights: their own linear layer (mma.sync over <= 8-token tiles)
  // bf16 row stride of the decode kernel's [out][H] matrices (rows padded to 2H + 16 bytes);
  // with 4-bit weights the lambda below turns 2H into the super-block row bytes
  const long long ldw_dec = q4 ? 2LL * H : static_cast<long long>(b.row_bytes);
  // ldw is the bf16 row stride; 4-bit rows take (K / 256) * 144 bytes plus the same tail
  auto linear = [&](const void* w, long long ldw, int N, int K, float* out, long long ldc, int acc) {
    if (e != cudaSuccess) return;
    if (q4) {
      e = launch_q4_linear(pf.xhi, pf.xlo, w, q4_row_bytes(K) + (ldw - 2LL * K), out, ldc, T, N, K, acc, pf.splitk,
                           kSplitKFloats, s);
    } else if (T <= 8) {
      e = launch_bf16_linear(pf.xhi, pf.xlo, w, ldw, out, ldc, T, N, K, acc, pf.splitk, kSplitKFloats, s);
    } else {
      LinearArgs a{pf.xhi, pf.xlo, w, ldw, out, ldc, T, N, K, acc, b.err, pf.splitk, kSplitKFloats};
      e = launch_linear(a, s);
    }
    ++m->launches;
  };
  if (q4)
    embed_rows_q4<<<T, kPT, 0, s>>>(tok, T, b.embed, b.row_bytes, H, c.vocab, pf.h, b.err);
  else
    embed_rows<<<T, kPT, 0, s>>>(tok, T, reinterpret_cast<const uint16_t*>(b.embed), b.row_bytes / 2, H, c.vocab,
                                  pf.h, b.err);
  chk();
  int di = 0, ai = 0;
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
    const LayerW& L = m->layers_host[l];
    const mk_prefill_layer& PL = m->pf_layers[l];
    rms_split<<<T, rms_threads(T), 0, s>>>(pf.h, H, L.norm1, b.eps, pf.xhi, pf.xlo);
    chk();
    if (L.kind == kDeltaNet) {
      const int rows = C + 2 * Hd;
      float* S = b.S + static_cast<size_t>(di) * Hd * dv * dk;
      float* ring = b.conv_ring + static_cast<size_t>(di) * Wc * C;
      ++di;
      linear(L.w_in, 2LL * H + 16, rows, H, pf.z, rows, 0);
      if (C % 128 == 0 && (dk == 64 || dk == 128) && rows % 4 == 0 && Wc <= kPrepMaxConv) {
        dn_prep_v4<<<dim3((T + 8 * kPrepTokensPerWarp - 1) / (8 * kPrepTokensPerWarp), C / 128 + 1), 256, 0, s>>>(
            pf.z, rows, T, b.pos, off, ring, Wc, C, Hd, dk, L.conv, pf.y, rows);
      } else if (T <= 64) {   // few tokens: a (token, vector) grid keeps the GPU busy
        dn_prep_wide<<<dim3(T, 2 * Hd + (Hd * dv + 127) / 128 + 1), 128, 0, s>>>(pf.z, rows, b.pos, off, ring, Wc, C,
                                                                                Hd, dk, dv, L.conv, pf.y, rows);
      } else {
        dn_prep<<<T, kPT, C * sizeof(float), s>>>(pf.z, rows, b.pos, off, ring, Wc, C, Hd, dk, L.conv, pf.y, rows);
      }
      chk();
      WyBufs wy{pf.y, rows, pf.u, pf.w, pf.p, pf.gam, pf.dec, pf.o, T, Hd, dk, dv, nullptr, nullptr, nullptr, 0};
      if (vs) {
        const size_t r = static_cast<size_t>(vs->rows) * (di - 1);
        if (e == cudaSuccess)
          e = cudaMemcpy2DAsync(vs->raw + r * C, C * sizeof(float), pf.z, rows * sizeof(float), C * sizeof(float), T,
                                cudaMemcpyDeviceToDevice, s);
        wy.save_g = vs->g + r * Hd;
        wy.save_k = vs->k + r * Hd * dk;
        wy.save_delta = vs->delta + r * Hd * dv;
        wy.keep_state = 1;
      } else {
        conv_history_update<<<dim3((C + kPT - 1) / kPT, Wc - 1), kPT, 0, s>>>(pf.z, rows, T, b.pos, off, ring, Wc, C);
        chk();
      }
      const int nch = (T + kChunk - 1) / kChunk;
      // two or more chunks of a prompt: the state pass on the tensor cores
      const bool tcs = !vs && pf.img && nch >= 2 && nch <= 128 && dk == dv && (dk == 128 || dk == 64) && rows % 4 == 0;
      if (tcs) {
        wy.img = pf.img;
        wy.err = b.err;
        if (dk == 128) {
          wy_prep_tc<128, 128><<<dim3(nch, Hd), 128, kWyPrepTcSmem, s>>>(wy);
          chk();
          wy_state_tc<128, 128><<<dim3(Hd, dv / kRowGroup), 128, wy_tc_smem<128>(), s>>>(wy, S);
        } else {
          wy_prep_tc<64, 64><<<dim3(nch, Hd), 128, kWyPrepTcSmem, s>>>(wy);
          chk();
          wy_state_tc<64, 64><<<dim3(Hd, dv / kRowGroup), 128, wy_tc_smem<64>(), s>>>(wy, S);
        }
      } else if (dk == 128 && dv == 128 && rows % 4 == 0) {   // 16-byte rows of q, k
        wy_prep_fast<128, 128><<<dim3(nch, Hd), 256, wy_fast_smem<128, 128>(false), s>>>(wy);
        chk();
        wy_state_fast<128, 128><<<dim3(Hd, dv / kRowGroup), 256, wy_fast_smem<128, 128>(true), s>>>(wy, S);
      } else if (dk == 64 && dv == 64 && rows % 4 == 0) {
        wy_prep_fast<64, 64><<<dim3(nch, Hd), 256, wy_fast_smem<64, 64>(false), s>>>(wy);
        chk();
        wy_state_fast<64, 64><<<dim3(Hd, dv / kRowGroup), 256, wy_fast_smem<64, 64>(true), s>>>(wy, S);
      } else {
        wy_prep<<<dim3(nch, Hd), 256, wy_prep_smem(dk, dv), s>>>(wy);
        chk();
        wy_state<<<dim3(Hd, dv / kRowGroup), 256, wy_state_smem(dk), s>>>(wy, S);
      }
      chk();
      gate_split<<<dim3(T, (Hd * dv + 1023) / 1024), kPT, 0, s>>>(pf.o, Hd * dv, nullptr, 0, Hd * dv, pf.xhi, pf.xlo);
      chk();
      linear(q4 ? L.w_out_q4 : PL.w_out, 2LL * Hd * dv, H, Hd * dv, pf.h, H, 1);
    } else {
      const int rows = b.at_in_rows;
      uint16_t* kc = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(b.kc) +
                                                 static_cast<size_t>(ai) * Hkv * c.max_ctx * b.kv_rb);
      uint16_t* vc = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(b.vc) +
                                                 static_cast<size_t>(ai) * Hkv * c.max_ctx * b.kv_rb);
      ++ai;
      linear(L.w_in, ldw_dec, rows, H, pf.z, rows, 0);
      at_prep<<<T, kPT, b.kv_q8 ? 2 * static_cast<size_t>(Hkv) * D * sizeof(float) : 0, s>>>(
          pf.z, rows, b.pos, off, b.inv_freq, Hq, Hkv, D, c.at_out_gate, kc, vc, c.max_ctx, pf.y, qd, b.kv_rb, b.kv_q8);
      chk();
      const long long nk_gemm = (m->pos_max + off + T + 63) / 64 * 64;   // covers every key of the pass
      if (b.kv_q8 && e == cudaSuccess) {   // the attention kernels below read bf16 rows
        const int nrows = static_cast<int>(std::min<long long>(nk_gemm, c.max_ctx));
        kv_dequant_bf16<<<dim3(nrows, Hkv, 2), 64, 0, s>>>(reinterpret_cast<const uint8_t*>(kc),
                                                           reinterpret_cast<const uint8_t*>(vc), Hkv, D, c.max_ctx,
                                                           b.kv_rb, b.pos, off + T - 1, pf.kvd);
        chk();
        kc = pf.kvd;
        vc = pf.kvd + static_cast<size_t>(Hkv) * c.max_ctx * D;
      }
      if (T >= kFlashAttnMinRows && pf.vt && nk_gemm <= pf.nk_max) {
        // flash attention on the tensor cores: V^T of every kv head, the queries of every
        // head as bf16 high / low parts, then one launch over (query tile, head)
        const int nk = static_cast<int>(nk_gemm);
        for (int g = 0; g < Hkv && e == cudaSuccess; ++g) {
          v_transpose<<<dim3(nk / 32, (D + 31) / 32), dim3(32, 8), 0, s>>>(
              vc + static_cast<size_t>(g) * c.max_ctx * D, D, nk, b.pos, off + T - 1, c.max_ctx,
              pf.vt + static_cast<size_t>(g) * D * nk);
          chk();
        }
        if (e == cudaSuccess) {
          e = launch_split_bf16(pf.y, qd, pf.xhi, pf.xlo, T, qd, s);
          ++m->launches;
        }
        if (e == cudaSuccess) {
          e = launch_attn_flash(pf.xhi, pf.xlo, kc, pf.vt, b.pos, off, T, Hq, Hkv, D, c.max_ctx, nk, pf.o, qd,
                                pf.flash_items, b.err, s);
          ++m->launches;
        }
      } else {
        // key splits when T * Hkv CTAs would leave most of the GPU idle (verify passes, short prompts)
        int nsplit = 1;
        if (T * Hkv < 148 && T <= kAttnSplitRows) nsplit = std::min(kAttnMaxSplit, (296 + T * Hkv - 1) / (T * Hkv));
        attn_prefill<<<dim3(T, Hkv, nsplit), 256, attn_prefill_smem(Hq / Hkv, D), s>>>(
            pf.y, qd, kc, vc, b.pos, off, Hq, Hkv, D, c.max_ctx, pf.o, qd, nsplit, pf.apart);
        chk();
        if (nsplit > 1) {
          attn_combine<<<dim3(T, Hq), std::min(D, 256), 0, s>>>(pf.apart, nsplit, Hq, D, pf.o, qd);
          chk();
        }
      }
      gate_split<<<dim3(T, (qd + 1023) / 1024), kPT, 0, s>>>(pf.o, qd, c.at_out_gate ? pf.z + qd : nullptr, rows, qd,
                                                             pf.xhi, pf.xlo);
      chk();
      linear(q4 ? L.w_out_q4 : PL.w_out, 2LL * qd, H, qd, pf.h, H, 1);
    }
    if (e != cudaSuccess) break;
    rms_split<<<T, rms_threads(T), 0, s>>>(pf.h, H, L.norm2, b.eps, pf.xhi, pf.xlo);
    chk();
    if (!q4 && PL.w_gu && T > 128 && F % 64 == 0) {
      // gate and up in one GEMM whose epilogue writes SiLU(gate) * up as bf16 high / low parts
      // (into the projection buffer, which holds 2 T F floats); the down-projection reads them
      uint16_t* ahi = reinterpret_cast<uint16_t*>(pf.z);
      uint16_t* alo = ahi + static_cast<size_t>(T) * F;
      if (e == cudaSuccess) {
        LinearArgs a{pf.xhi, pf.xlo, PL.w_gu, 2LL * H, pf.z, 2LL * F, T, 2 * F, H, 0, b.err};
        a.act_hi = ahi;
        a.act_lo = alo;
        e = launch_linear(a, s);
        ++m->launches;
      }
      if (e == cudaSuccess) {
        LinearArgs a{ahi, alo, PL.w_down, 2LL * F, pf.h, H, T, H, F, 1, b.err, pf.splitk, kSplitKFloats};
        e = launch_linear(a, s);
        ++m->launches;
      }
    } else {
      linear(L.w_gate, ldw_dec, F, H, pf.z, 2LL * F, 0);
      linear(L.w_up, ldw_dec, F, H, pf.z + F, 2LL * F, 0);
      act_split<<<dim3(T, (F + 1023) / 1024), kPT, 0, s>>>(pf.z, F, pf.xhi, pf.xlo);
      chk();
      linear(q4 ? L.w_down_q4 : PL.w_down, 2LL * F, H, F, pf.h, H, 1);
    }
  }
  return e;
}

}  // namespace

cudaError_t set_prefill_smem_limits() {
  static std::atomic<uint64_t> done{0};   // per device
  return once_per_device(done, [] {
    cudaError_t e = cudaFuncSetAttribute(wy_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(wy_state, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(dn_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(wy_prep_fast<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(wy_state_fast<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(wy_prep_fast<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(wy_state_fast<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bf16_linear_mma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(4 * kBfDepth * 32 * 128));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(q4_linear_mma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(4 * kQ4Depth * 32 * 144));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wy_state_tc<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(wy_tc_smem<128>()));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wy_state_tc<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(wy_tc_smem<64>()));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wy_prep_tc<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kWyPrepTcSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wy_prep_tc<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kWyPrepTcSmem));
    return e;
  });
}

size_t prefill_smem_need(int dk, int dv, int grp, int D, int C) {
  size_t n = std::max(wy_prep_smem(dk, dv), wy_state_smem(dk));
  n = std::max(n, attn_prefill_smem(grp, D));
  return std::max(n, static_cast<size_t>(C) * sizeof(float));
}

}  // namespace mk

int mk_prefill_batched(mk_model* m, const int32_t* d_tokens, int n, cudaStream_t s) {
  const mk::DecodeParams& b = m->base;
  cudaError_t e = mk::set_prefill_smem_limits();
  if (e == cudaSuccess) {
    mk::check_capacity<<<1, 1, 0, s>>>(b.pos, n, m->cfg.max_ctx, b.err);
    e = cudaGetLastError();
    ++m->launches;
  }
  for (int off = 0; off < n && e == cudaSuccess; off += m->pf.rows) {
    const int T = std::min(m->pf.rows, n - off);
    e = mk::prefill_pass(m, d_tokens + off, T, off, s);
  }
  if (e == cudaSuccess) {
    mk::advance_pos<<<1, 1, 0, s>>>(b.pos, n, m->cfg.max_ctx);
    e = cudaGetLastError();
    ++m->launches;
  }
  if (e != cudaSuccess) {
    mk_set_last_error(std::string("batched prefill: ") + cudaGetErrorString(e));
    return MK_ERR_CUDA;
  }
  m->pos_hint += n;
  m->pos_max += n;
  return MK_OK;
}

// After a batched prefill of n tokens: the final RMSNorm of the last token's residual row (row
// (n - 1) mod rows of the last pass), the tied LM head over that one row on the tensor cores,
// and its greedy token; logits into d_logits (or the projection scratch when it is null).
int mk_prefill_tail(mk_model* m, int n, float* d_logits, int32_t* d_next_token, cudaStream_t s) {
  const mk::DecodeParams& b = m->base;
  const mk_config& c = m->cfg;
  const int rows = m->pf.rows;
  const int r = (n - 1) % rows;
  float* logits = d_logits ? d_logits : m->pf.z;
  cudaError_t e = cudaSuccess;
  mk::rms_split<<<1, mk::rms_threads(1), 0, s>>>(m->pf.h + static_cast<size_t>(r) * c.hidden, c.hidden, b.norm_f, b.eps,
                                                  m->pf.xhi, m->pf.xlo);
  e = cudaGetLastError();
  ++m->launches;
  if (e == cudaSuccess) {
    e = b.q4 ? mk::launch_q4_linear(m->pf.xhi, m->pf.xlo, b.embed, b.row_bytes, logits, c.vocab, 1, c.vocab, c.hidden, 0,
                                    m->pf.splitk, mk::kSplitKFloats, s)
             : mk::launch_bf16_linear(m->pf.xhi, m->pf.xlo, b.embed, b.row_bytes, logits, c.vocab, 1, c.vocab, c.hidden,
                                      0, m->pf.splitk, mk::kSplitKFloats, s);
    ++m->launches;
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(m->pf.best, 0, sizeof(unsigned long long), s);
  if (e == cudaSuccess) {
    mk::row_argmax<<<dim3(1, 64), 256, 0, s>>>(logits, c.vocab, m->pf.best);
    e = cudaGetLastError();
    ++m->launches;
  }
  if (e == cudaSuccess && d_next_token) {
    mk::argmax_token<<<1, 1, 0, s>>>(m->pf.best, d_next_token);
    e = cudaGetLastError();
    ++m->launches;
  }
  if (e != cudaSuccess) {
    mk_set_last_error(std::string("prefill logits: ") + cudaGetErrorString(e));
    return MK_ERR_CUDA;
  }
  return MK_OK;
}

// One verify pass on stream s (every launch; no host-side bookkeeping of the position).
static int verify_pass(mk_model* m, const int32_t* d_tokens, int K, int32_t* d_n_accepted, int32_t* d_out_tokens,
                       float* d_logits, cudaStream_t s, float temperature, const float* d_uniforms) {
  const mk::DecodeParams& b = m->base;
  const mk_config& c = m->cfg;
  const int T = K + 1;
  const mk_verify_ws& vs = m->vf;
  cudaError_t e = mk::set_prefill_smem_limits();
  auto chk = [&]() {
    if (e == cudaSuccess) e = cudaGetLastError();
    ++m->launches;
  };
  if (e == cudaSuccess) {
    mk::check_capacity<<<1, 1, 0, s>>>(b.pos, T, c.max_ctx, b.err);
    chk();
  }
  // 1. every layer over the K + 1 tokens, one pass over the weights
  if (e == cudaSuccess) e = mk::prefill_pass(m, d_tokens, T, 0, s, &vs);
  // 2. final norm, LM head on the tensor cores for all K + 1 positions, greedy tokens
  float* logits = d_logits ? d_logits : vs.logits;
  if (e == cudaSuccess) {
    mk::rms_split<<<T, mk::rms_threads(T), 0, s>>>(m->pf.h, c.hidden, b.norm_f, b.eps, m->pf.xhi, m->pf.xlo);
    chk();
  }
  if (e == cudaSuccess && b.q4) {   // 4-bit tied LM head
    e = mk::launch_q4_linear(m->pf.xhi, m->pf.xlo, b.embed, b.row_bytes, logits, c.vocab, T, c.vocab, c.hidden, 0,
                             m->pf.splitk, mk::kSplitKFloats, s);
    ++m->launches;
  } else if (e == cudaSuccess && T <= 8) {   // bf16 tied LM head, few tokens
    e = mk::launch_bf16_linear(m->pf.xhi, m->pf.xlo, b.embed, b.row_bytes, logits, c.vocab, T, c.vocab, c.hidden, 0,
                               m->pf.splitk, mk::kSplitKFloats, s);
    ++m->launches;
  } else if (e == cudaSuccess) {
    mk::LinearArgs a{m->pf.xhi, m->pf.xlo, b.embed, b.row_bytes, logits, c.vocab, T, c.vocab, c.hidden, 0, b.err};
    e = mk::launch_linear(a, s);
    ++m->launches;
  }
  if (d_uniforms) {
    // 3'. sampled acceptance: per-slice row statistics, the draft tests, the chunk sums of
    // the stopping row, the draw
    double* part = vs.stats;
    SampDecision* dec = reinterpret_cast<SampDecision*>(part + static_cast<size_t>(vs.rows) * kSampSlices * 2);
    double* csum = reinterpret_cast<double*>(dec + 1);
    const double inv_tau = 1.0 / static_cast<double>(temperature);
    if (e == cudaSuccess) {
      mk::row_softmax_partials<<<dim3(T, kSampSlices), mk::kSampThreads, 0, s>>>(logits, c.vocab, inv_tau, part);
      chk();
    }
    if (e == cudaSuccess) {
      mk::samp_decide<<<1, 32, 0, s>>>(d_tokens, K, logits, c.vocab, inv_tau, part, d_uniforms, dec);
      chk();
    }
    if (e == cudaSuccess) {
      mk::samp_chunk_sums<<<kDrawChunks / mk::kSampThreads, mk::kSampThreads, 0, s>>>(logits, c.vocab, inv_tau, dec,
                                                                                      csum);
      chk();
    }
    if (e == cudaSuccess) {
      mk::samp_select<<<1, 32, 0, s>>>(d_tokens, logits, c.vocab, inv_tau, dec, csum, d_uniforms, m->ws_n,
                                       d_n_accepted, d_out_tokens);
      chk();
    }
  } else {
    if (e == cudaSuccess) e = cudaMemsetAsync(m->pf.best, 0, sizeof(unsigned long long) * T, s);
    if (e == cudaSuccess) {
      mk::row_argmax<<<dim3(T, 64), 256, 0, s>>>(logits, c.vocab, m->pf.best);
      chk();
    }
    // 3. longest matching prefix plus the bonus token
    if (e == cudaSuccess) {
      mk::accept_prefix<<<1, 32, 0, s>>>(d_tokens, m->pf.best, K, m->ws_n, d_n_accepted, d_out_tokens, vs.greedy);
      chk();
    }
  }
  // 4. commit: DeltaNet states and conv histories of the accepted prefix, then the position
  int di = 0;
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
    if (c.pattern[l] != 'D') continue;
    const size_t r = static_cast<size_t>(vs.rows) * di;
    float* S = b.S + static_cast<size_t>(di) * c.dn_heads * c.dn_dv * c.dn_dk;
    float* ring = b.conv_ring + static_cast<size_t>(di) * c.conv_width * b.C;
    mk::commit_state<<<dim3(c.dn_heads, c.dn_dv / mk::kRowGroup), 256, 0, s>>>(
        S, vs.delta + r * c.dn_heads * c.dn_dv, vs.k + r * c.dn_heads * c.dn_dk, vs.g + r * c.dn_heads, m->ws_n,
        c.dn_heads, c.dn_dk, c.dn_dv);
    chk();
    mk::commit_conv<<<dim3((b.C + 255) / 256, c.conv_width - 1), 256, 0, s>>>(vs.raw + r * b.C, ring, c.conv_width,
                                                                               b.C, b.pos, m->ws_n);
    chk();
    ++di;
  }
  if (e == cudaSuccess) {
    mk::advance_pos_accepted<<<1, 1, 0, s>>>(b.pos, m->ws_n, c.max_ctx);
    chk();
  }
  if (e != cudaSuccess) {
    mk_set_last_error(std::string("verify pass: ") + cudaGetErrorString(e));
    return MK_ERR_CUDA;
  }
  return MK_OK;
}

// Verify passes with the output arguments of the previous one replay a CUDA graph of the ~10
// launches per layer (the first pass with new arguments runs uncaptured, so every lazy setup is
// done; the second is captured and replayed). The drafts are first copied into the model's
// own token buffer, so every launch argument of a pass is fixed by the model, K and the output
// arguments; the device position is read by the kernels. Models with the 8-bit KV cache size one
// launch from the host's bound of the position, so they always run uncaptured.
int mk_verify_batched(mk_model* m, const int32_t* d_tokens, int K, int32_t* d_n_accepted, int32_t* d_out_tokens,
                      float* d_logits, cudaStream_t s, float temperature, const float* d_uniforms) {
  const int T = K + 1;
  int rc = MK_OK;
  mk_verify_graph& g = m->vgraph;
  // the pass reads the tokens from the model's own buffer (ws_g, max_draft + 1 entries), so a
  // new token array does not need a new graph
  if (cudaMemcpyAsync(m->ws_g, d_tokens, sizeof(int32_t) * T, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    mk_set_last_error("verify pass: token copy failed");
    return MK_ERR_CUDA;
  }
  d_tokens = m->ws_g;
  const bool same = g.tokens == d_tokens && g.K == K && g.n_accepted == d_n_accepted && g.out_tokens == d_out_tokens &&
                    g.logits == d_logits && g.temperature == temperature && g.uniforms == d_uniforms;
  if (!same) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    g.exec = nullptr;
    g.tokens = d_tokens;
    g.K = K;
    g.n_accepted = d_n_accepted;
    g.out_tokens = d_out_tokens;
    g.logits = d_logits;
    g.temperature = temperature;
    g.uniforms = d_uniforms;
    g.seen = 0;
  }
  const bool capturable = m->cfg.kv_format == MK_KV_BF16 && mk::set_prefill_smem_limits() == cudaSuccess;
  if (!capturable || (!g.exec && g.seen == 0)) {
    rc = verify_pass(m, d_tokens, K, d_n_accepted, d_out_tokens, d_logits, s, temperature, d_uniforms);
    g.seen = 1;
  } else {
    cudaError_t e = cudaSuccess;
    if (!g.stream) e = cudaStreamCreateWithFlags(&g.stream, cudaStreamNonBlocking);
    if (e == cudaSuccess && !g.ev_in) e = cudaEventCreateWithFlags(&g.ev_in, cudaEventDisableTiming);
    if (e == cudaSuccess && !g.ev_out) e = cudaEventCreateWithFlags(&g.ev_out, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(g.ev_in, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(g.stream, g.ev_in, 0);
    if (e == cudaSuccess && !g.exec) {   // capture this pass
      e = cudaStreamBeginCapture(g.stream, cudaStreamCaptureModeThreadLocal);
      if (e == cudaSuccess) {
        const int64_t l0 = m->launches;
        const int prc = verify_pass(m, d_tokens, K, d_n_accepted, d_out_tokens, d_logits, g.stream, temperature,
                                    d_uniforms);
        cudaGraph_t graph = nullptr;
        e = cudaStreamEndCapture(g.stream, &graph);
        if (prc != MK_OK) {
          if (graph) cudaGraphDestroy(graph);
          return prc;
        }
        if (e == cudaSuccess) e = cudaGraphInstantiate(&g.exec, graph, 0);
        if (graph) cudaGraphDestroy(graph);
        g.launches = m->launches - l0;
        m->launches = l0;
      }
    }
    if (e == cudaSuccess) e = cudaGraphLaunch(g.exec, g.stream);
    if (e == cudaSuccess) e = cudaEventRecord(g.ev_out, g.stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, g.ev_out, 0);
    if (e != cudaSuccess) {
      mk_set_last_error(std::string("verify pass (graph): ") + cudaGetErrorString(e));
      return MK_ERR_CUDA;
    }
    m->launches += g.launches;
  }
  if (rc != MK_OK) return rc;
  m->pos_hint += 1;   // at least one position is always committed; the exact count is on the device
  m->pos_max += T;
  return MK_OK;
}
