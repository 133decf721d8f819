// Linear layers of the prefill on the sm_100a tensor cores.
//
//   C[m][n] (+)= sum_k X[m][k] * W[n][k]      (m < M tokens, n < N features, k < K)
//
// X arrives as fp32 and is split into bf16 high and low parts (X = Xhi + Xlo up to the
// rounding of Xlo, about 16 bits of X's mantissa kept); W is bf16. Both parts multiply
// the same W tile into one fp32 accumulator in tensor memory, so the product carries
// the activations at about fp32 precision, the same precision the decode megakernel
// keeps its activations at.
//
// One CTA computes one 128 x BN tile of C:
// persistent CTAs (at most one per SM) walk the tiles (and K splits):
//   warp 0   allocates 2 x BN TMEM columns (two accumulators); its lane 0 is the TMA
//            producer: per 64-wide K block it loads Xhi, Xlo [128 x 64] and W [BN x 64]
//            (128-byte swizzled) into a 3-4 stage shared-memory ring;
//   warp 1   lane 0 issues tcgen05.mma (M = 128, N = BN, K = 16; 8 per K block) into the
//            tile's accumulator, commits each stage back to the producer and the finished
//            accumulator to the epilogue;
//   warps 2-5 read the accumulator rows from TMEM (warp w owns lanes 32 (w % 4) ..), store
//            (or add into) C, and hand the accumulator back, while the next tile's MMAs run
//            in the other one.
// Every wait has a time limit; on expiry the CTA latches an error bit and winds down.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "mk_model.h"
#include "tc.cuh"

#include <cudaTypedefs.h>

namespace mk {

namespace {

constexpr uint64_t kGemmWaitNs = 1000000000ull;
constexpr int kBM = 128, kBK = 64;

template <int BN>
struct GemmShape {
  static constexpr int kStages = BN >= 256 ? 3 : 4;
  static constexpr int kABytes = kBM * kBK * 2;        // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = 2 * kABytes + kBBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = kRingBytes + 256 + 1024;   // + barriers, + alignment slack
};

struct GemmBars {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t acc_full[2];    // accumulator buffer b holds a finished tile
  uint64_t acc_empty[2];   // the epilogue has drained buffer b
  uint32_t tmem;
  int abort;
};

// Persistent: CTA c walks the work items c, c + grid, ... (item = (N tile, M tile, K split)),
// with two TMEM accumulators so that the epilogue of one item overlaps the MMAs of the next.
template <int BN>
__global__ void __launch_bounds__(192, 1)
    linear_kernel(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
                  const __grid_constant__ CUtensorMap tb, float* __restrict__ C, long long ldc, int M, int N, int K,
                  int accumulate, int* err, float* __restrict__ ws, int nz, uint16_t* __restrict__ act_hi,
                  uint16_t* __restrict__ act_lo) {
  using S = GemmShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmBars* gb = reinterpret_cast<GemmBars*>(smem + S::kRingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (N + BN - 1) / BN, tiles_m = (M + kBM - 1) / kBM;
  const int items = tiles_n * tiles_m * nz;
  const int nkall = K / kBK;
  auto a_hi = [&](int s) { return smem + s * S::kStageBytes; };
  auto a_lo = [&](int s) { return smem + s * S::kStageBytes + S::kABytes; };
  auto b_t = [&](int s) { return smem + s * S::kStageBytes + 2 * S::kABytes; };
  // item -> tile origin and K-block range (split z takes [kb0, kb1))
  auto decode = [&](int w, int& n0, int& m0, int& z, int& kb0, int& kb1) {
    const int tn = w % tiles_n, rest = w / tiles_n;
    n0 = tn * BN;
    m0 = (rest % tiles_m) * kBM;
    z = rest / tiles_m;
    kb0 = static_cast<int>((static_cast<long long>(nkall) * z) / nz);
    kb1 = static_cast<int>((static_cast<long long>(nkall) * (z + 1)) / nz);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&gb->full[s], 1);
      mbar_init(&gb->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&gb->acc_full[b], 1);
      mbar_init(&gb->acc_empty[b], 4);   // one arrival per epilogue warp
    }
    gb->abort = 0;
    fence_barrier_init();
    tc::prefetch_tensormap(&ta_hi);
    tc::prefetch_tensormap(&ta_lo);
    tc::prefetch_tensormap(&tb);
  }
  if (warp == 0) {
    tc::tmem_alloc(&gb->tmem, 2 * BN);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = gb->tmem;
  volatile int* abort = &gb->abort;

  if (warp == 0) {
    if (lane == 0) {   // ---- TMA producer: one running K-block counter over all items
      uint32_t kc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
        int n0, m0, z, kb0, kb1;
        decode(w, n0, m0, z, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++kc) {
          const int s = kc % S::kStages;
          if (kc >= static_cast<uint32_t>(S::kStages) &&
              !mbar_wait(&gb->empty[s], ((kc / S::kStages) - 1) & 1, abort, kGemmWaitNs)) {
            if (!*abort) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
            *abort = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&gb->full[s], S::kStageBytes);
          tc::tma_load_2d(a_hi(s), &ta_hi, kb * kBK, m0, &gb->full[s]);
          tc::tma_load_2d(a_lo(s), &ta_lo, kb * kBK, m0, &gb->full[s]);
          tc::tma_load_2d(b_t(s), &tb, kb * kBK, n0, &gb->full[s]);
        }
      }
      int never = 0;   // let the copies this lane issued land before the CTA ends (bounded)
      for (uint32_t k = kc > static_cast<uint32_t>(S::kStages) ? kc - S::kStages : 0; k < kc; ++k)
        mbar_wait(&gb->full[k % S::kStages], (k / S::kStages) & 1, &never, kGemmWaitNs / 5);
    }
  } else if (warp == 1) {
    if (lane == 0) {   // ---- MMA issuer
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kBM, BN);
      uint32_t kc = 0;
      bool ok = true;
      int i = 0;
      for (int w = blockIdx.x; w < items && ok; w += gridDim.x, ++i) {
        int n0, m0, z, kb0, kb1;
        decode(w, n0, m0, z, kb0, kb1);
        const int buf = i & 1;
        if (i >= 2 && !mbar_wait(&gb->acc_empty[buf], ((i >> 1) - 1) & 1, abort, kGemmWaitNs)) {
          if (!*abort) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
          *abort = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++kc) {
          const int s = kc % S::kStages;
          if (!mbar_wait(&gb->full[s], (kc / S::kStages) & 1, abort, kGemmWaitNs)) {
            if (!*abort) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
            *abort = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = tc::desc_kmajor_sw128(b_t(s) + kk * 32);
            tc::mma_bf16(acc, tc::desc_kmajor_sw128(a_hi(s) + kk * 32), bd, idesc, (kb > kb0 || kk) ? 1u : 0u);
            tc::mma_bf16(acc, tc::desc_kmajor_sw128(a_lo(s) + kk * 32), bd, idesc, 1u);
          }
          tc::mma_commit(&gb->empty[s]);
        }
        tc::mma_commit(&gb->acc_full[buf]);   // arrives once every MMA issued so far has completed
      }
    }
  } else {   // ---- epilogue: warps 2..5
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int i = 0;
    for (int w = blockIdx.x; w < items; w += gridDim.x, ++i) {
      int n0, m0, z, kb0, kb1;
      decode(w, n0, m0, z, kb0, kb1);
      const int buf = i & 1;
      const bool okw = mbar_wait(&gb->acc_full[buf], (i >> 1) & 1, abort, kGemmWaitNs);
      tc::fence_after_sync();
      if (!okw && lane == 0) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
      if (!__all_sync(0xffffffffu, okw) || *abort) break;
      float* Cz = C;
      long long ldz = ldc;
      int accz = accumulate;
      if (nz > 1) {
        Cz = ws + static_cast<long long>(z) * M * N;
        ldz = N;
        accz = 0;
      }
      const int m = m0 + row;
      if (act_hi) {   // SwiGLU epilogue: gate columns pair with the up columns 64 to their right
        const uint32_t tbase = tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          if (((n0 + c0) & 127) >= 64) continue;
          float gv[16], uv[16];
          tc::tmem_ld16(tbase + c0, gv);
          tc::tmem_ld16(tbase + c0 + 64, uv);
          if (m < M && n0 + c0 + 64 < N) {
            const long long f = static_cast<long long>(m) * (N / 2) + ((n0 + c0) >> 7) * 64 + ((n0 + c0) & 63);
            uint32_t h[8], l[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float a0 = siluf_(gv[2 * j]) * uv[2 * j];
              const float a1 = siluf_(gv[2 * j + 1]) * uv[2 * j + 1];
              const uint16_t h0 = f_to_bf16(a0), h1 = f_to_bf16(a1);
              h[j] = h0 | (static_cast<uint32_t>(h1) << 16);
              l[j] = f_to_bf16(a0 - bf16_to_f(h0)) | (static_cast<uint32_t>(f_to_bf16(a1 - bf16_to_f(h1))) << 16);
            }
            uint4* dh = reinterpret_cast<uint4*>(act_hi + f);
            uint4* dl = reinterpret_cast<uint4*>(act_lo + f);
            dh[0] = make_uint4(h[0], h[1], h[2], h[3]);
            dh[1] = make_uint4(h[4], h[5], h[6], h[7]);
            dl[0] = make_uint4(l[0], l[1], l[2], l[3]);
            dl[1] = make_uint4(l[4], l[5], l[6], l[7]);
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&gb->acc_empty[buf]);
        continue;
      }
      float* crow = Cz + static_cast<long long>(m) * ldz + n0;
      const bool vec = (ldz % 4 == 0) && ((reinterpret_cast<uintptr_t>(Cz) & 15) == 0);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16];
        tc::tmem_ld16(tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
        if (m < M) {
          if (vec && n0 + c0 + 16 <= N) {
            float4* d4 = reinterpret_cast<float4*>(crow + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float4 o = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
              if (accz) {
                const float4 c = d4[j];
                o.x += c.x; o.y += c.y; o.z += c.z; o.w += c.w;
              }
              d4[j] = o;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n0 + c0 + j < N) crow[c0 + j] = accz ? crow[c0 + j] + v[j] : v[j];
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&gb->acc_empty[buf]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 2 * BN);
  }
}

// C[m][n] (+)= sum_z ws[z][m][n], z in order (deterministic).
__global__ void splitk_reduce(const float* __restrict__ ws, int nz, int M, int N, float* __restrict__ C, long long ldc,
                              int accumulate) {
  const long long total = static_cast<long long>(M) * N;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = i / N, n = i % N;
    float v = accumulate ? C[m * ldc + n] : 0.f;
    for (int z = 0; z < nz; ++z) v += ws[z * total + i];
    C[m * ldc + n] = v;
  }
}

__global__ void split_bf16_kernel(const float* __restrict__ x, long long ldx, uint16_t* __restrict__ hi,
                                  uint16_t* __restrict__ lo, int M, int K) {
  const long long total = static_cast<long long>(M) * K;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = i / K, k = i % K;
    const float v = x[m * ldx + k];
    const uint16_t h = f_to_bf16(v);
    hi[i] = h;
    lo[i] = f_to_bf16(v - bf16_to_f(h));
  }
}

// ---- host: tensor maps through the driver entry point (no link-time libcuda dependency)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 row-major [rows][cols] with a row stride of `stride_bytes`; box = 64 columns x box_rows.
bool make_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long stride_bytes,
              int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor maps are plain host structs that depend only on (base, rows, cols, stride, box);
// the prefill and verify passes reuse the same few hundred, so they are encoded once.
struct MapKey {
  const void* base;
  long long rows, cols, stride;
  int box;
  bool operator<(const MapKey& o) const {
    if (base != o.base) return base < o.base;
    if (rows != o.rows) return rows < o.rows;
    if (cols != o.cols) return cols < o.cols;
    if (stride != o.stride) return stride < o.stride;
    return box < o.box;
  }
};

bool cached_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long stride_bytes, int box) {
  static std::mutex mu;
  static std::map<MapKey, CUtensorMap> cache;
  const MapKey k{base, rows, cols, stride_bytes, box};
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(k);
  if (it != cache.end()) {
    *map = it->second;
    return true;
  }
  if (!make_map(map, base, rows, cols, stride_bytes, box)) return false;
  if (cache.size() > 65536) cache.clear();   // bound the cache (device buffers come and go)
  cache.emplace(k, *map);
  return true;
}

template <int BN>
cudaError_t launch_bn(const LinearArgs& a, cudaStream_t s) {
  using S = GemmShape<BN>;
  CUtensorMap ma_hi, ma_lo, mb;
  if (!cached_map(&ma_hi, a.x_hi, a.M, a.K, static_cast<long long>(a.K) * 2, kBM) ||
      !cached_map(&ma_lo, a.x_lo, a.M, a.K, static_cast<long long>(a.K) * 2, kBM) ||
      !cached_map(&mb, a.w, a.N, a.K, a.ldw_bytes, BN))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr_set{0};   // per device
  const cudaError_t attr = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(linear_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
  });
  if (attr != cudaSuccess) return attr;
  dim3 grid((a.N + BN - 1) / BN, (a.M + kBM - 1) / kBM);
  // split K when the tile grid leaves most SMs idle (few tokens) and the workspace holds it
  const int tiles = static_cast<int>(grid.x * grid.y), nk = a.K / kBK;
  int nz = 1;
  // few tokens (one M tile) and few N tiles: about one wave, >= 3 K blocks per CTA; a short
  // prompt (up to 8 M tiles) whose tile grid fills at most half the GPU: 2-4 splits of >= 8 K blocks
  if (a.ws && !a.act_hi && ((grid.y == 1 && tiles < 148 && nk >= 6) || (grid.y <= 8 && tiles <= 74 && nk >= 16))) {
    nz = grid.y == 1 ? std::min({(148 + tiles - 1) / tiles, nk / 3, 16}) : std::min({(148 + tiles - 1) / tiles, nk / 8, 4});
    const long long need = static_cast<long long>(a.M) * a.N;
    while (nz > 1 && need * nz > a.ws_floats) --nz;
  }
  const int items = tiles * nz;
  const int nctas = std::min(items, 148);
  linear_kernel<BN><<<nctas, 192, S::kSmemBytes, s>>>(ma_hi, ma_lo, mb, a.c, a.ldc, a.M, a.N, a.K, a.accumulate,
                                                      a.err, a.ws, nz, a.act_hi, a.act_lo);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && nz > 1) {
    const long long total = static_cast<long long>(a.M) * a.N;
    const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148 * 8));
    splitk_reduce<<<blocks, 256, 0, s>>>(a.ws, nz, a.M, a.N, a.c, a.ldc, a.accumulate);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

bool tensor_map_bf16(CUtensorMap* map, const void* base, long long rows, long long cols, long long stride_bytes,
                     int box_rows) {
  return cached_map(map, base, rows, cols, stride_bytes, box_rows);
}

cudaError_t launch_split_bf16(const float* x, long long ldx, uint16_t* hi, uint16_t* lo, int M, int K,
                              cudaStream_t s) {
  const long long total = static_cast<long long>(M) * K;
  if (total == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148 * 16));
  split_bf16_kernel<<<blocks, 256, 0, s>>>(x, ldx, hi, lo, M, K);
  return cudaGetLastError();
}

cudaError_t launch_linear(const LinearArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  if (a.K <= 0 || a.K % kBK != 0 || a.ldw_bytes % 16 != 0 || a.ldw_bytes < 2LL * a.K ||
      (reinterpret_cast<uintptr_t>(a.x_hi) & 15) || (reinterpret_cast<uintptr_t>(a.x_lo) & 15) ||
      (reinterpret_cast<uintptr_t>(a.w) & 15))
    return cudaErrorInvalidValue;
  if (a.act_hi && (a.N % 128 != 0 || !a.act_lo || (reinterpret_cast<uintptr_t>(a.act_hi) & 15) ||
                   (reinterpret_cast<uintptr_t>(a.act_lo) & 15)))
    return cudaErrorInvalidValue;
  // 256-wide tiles for many tokens and wide outputs, or whenever they still fill about a wave
  // (a 1024-wide output over thousands of tokens: 128 tiles of 256 in one wave rather than 256
  // tiles of 128 in 1.7); 128-wide for few tokens (more CTAs to split over)
  const long long tiles256 = static_cast<long long>((a.N + 255) / 256) * ((a.M + kBM - 1) / kBM);
  const bool wide = a.M > kBM && (a.N >= 2048 || tiles256 >= 120);
  return wide ? launch_bn<256>(a, s) : launch_bn<128>(a, s);
}

}  // namespace mk

// ---------------------------------------------------------------- C ABI
extern "C" int mk_linear(const float* d_x, int64_t ldx, int32_t M, int32_t K, const void* d_w, int64_t ldw_bytes,
                         int32_t N, float* d_c, int64_t ldc, int32_t accumulate, void* d_scratch, size_t scratch_bytes,
                         int32_t* d_err, void* stream) {
  if (!d_x || !d_w || !d_c || !d_err || !d_scratch) {
    mk_set_last_error("mk_linear: NULL pointer");
    return MK_ERR_ARG;
  }
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || ldx < K || ldc < N || ldw_bytes < 2LL * K || ldw_bytes % 16 != 0) {
    mk_set_last_error("mk_linear: bad sizes (K must be a positive multiple of 64, ldw_bytes a multiple of 16 "
                      "and >= 2K, ldx >= K, ldc >= N)");
    return MK_ERR_ARG;
  }
  if (scratch_bytes < 4ull * static_cast<unsigned long long>(M) * K) {
    mk_set_last_error("mk_linear: scratch must hold 4*M*K bytes");
    return MK_ERR_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(d_w) & 15) || (reinterpret_cast<uintptr_t>(d_scratch) & 15)) {
    mk_set_last_error("mk_linear: d_w and d_scratch must be 16-byte aligned");
    return MK_ERR_ARG;
  }
  if (M == 0 || N == 0) return MK_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* hi = static_cast<uint16_t*>(d_scratch);
  uint16_t* lo = hi + static_cast<size_t>(M) * K;
  cudaError_t e = mk::launch_split_bf16(d_x, ldx, hi, lo, M, K, s);
  if (e == cudaSuccess) {
    mk::LinearArgs a{hi, lo, d_w, ldw_bytes, d_c, ldc, M, N, K, accumulate ? 1 : 0, d_err};
    e = mk::launch_linear(a, s);
  }
  if (e != cudaSuccess) {
    mk_set_last_error(std::string("mk_linear: ") + cudaGetErrorString(e));
    return MK_ERR_CUDA;
  }
  return MK_OK;
}
