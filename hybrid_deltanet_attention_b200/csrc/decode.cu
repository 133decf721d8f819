// Persistent decode megakernel: one launch runs every layer of one batch-1 forward step.
//
// Design (the Hacker News post on the fused Qwen3.5-0.8B kernel, design bullets,
// is the prior art: one launch per token, persistent blocks on every SM, a grid-wide
// barrier instead of kernel boundaries; re-done here for sm_100a):
//  * grid = one CTA per SM (cooperative launch, so all CTAs are co-resident);
//  * each CTA owns a fixed contiguous slice of every weight matrix; a producer warp
//    streams the CTA's whole per-step weight sequence through a 6 x 32 KB shared-memory
//    ring with cp.async.bulk, independent of the grid barriers, so HBM stays busy while
//    the consumer warps wait at a barrier;
//  * 8 consumer warps do the arithmetic in fp32 from shared memory;
//  * out-projections and the MLP down-projection are split over their input dim
//    (split-K) and accumulated into the residual with vector atomics, so a DeltaNet
//    layer needs 3 grid barriers and an attention layer 4;
//  * every wait (grid barrier, pipeline slot) has a time limit; on expiry the kernel
//    latches a bit in the device error word and every CTA returns.
#include "dev.cuh"
#include "mk_internal.h"
#include "../../include/mk.h"

namespace mk {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: a healthy wait takes microseconds
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 200 ms for in-flight copies to land
constexpr int kMaxGroups = 8;                      // float4 groups per thread: H <= 8192

enum Phase : int { kPhIn = 0, kPhMix = 1, kPhAttOut = 2, kPhMlp = 3, kPhFinal = 4 };

struct Seg {
  const uint8_t* src;
  int rows;
  int row_bytes;
};

struct __align__(16) Shared {
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  int abort_flag;      // set by any thread that gives up a wait
  int decision;        // consumer-wide abort decision, written only inside grid_barrier
  int tok;
  int pos;
  int bad;
  float red[kConsumerWarps];
  float best_v[kConsumerWarps];
  int best_i[kConsumerWarps];
};

__device__ __forceinline__ void split_range(int n, int c, int G, int& b, int& e) {
  b = static_cast<int>((static_cast<long long>(n) * c) / G);
  e = static_cast<int>((static_cast<long long>(n) * (c + 1)) / G);
}

__device__ __forceinline__ void attn_split(int n, int G, int Hkv, int max_splits, int& CH, int& nsplit) {
  int per = G / Hkv;
  if (per < 1) per = 1;
  if (per > max_splits) per = max_splits;
  int ch = (n + per - 1) / per;
  if (ch < kAttnMinChunk) ch = kAttnMinChunk;
  ch = (ch + 15) / 16 * 16;
  CH = ch;
  nsplit = (n + ch - 1) / ch;
}

// The weight (and DeltaNet-state) rows a CTA streams in one phase. Producer and
// consumers both call this, so they agree on the chunk sequence.
__device__ int phase_segments(const DecodeParams& p, const LayerW& L, int phase, int cta, int G, Seg* s) {
  const int rb = p.row_bytes;
  int b, e, n = 0;
  switch (phase) {
    case kPhIn: {
      const int rows = (L.kind == kDeltaNet) ? (p.C + 2 * p.Hd) : p.at_in_rows;
      split_range(rows, cta, G, b, e);
      if (e > b) s[n++] = {L.w_in + static_cast<size_t>(b) * rb, e - b, rb};
      break;
    }
    case kPhMix: {
      if (L.kind != kDeltaNet) break;
      split_range(p.Hd * p.dv, cta, G, b, e);
      if (e > b) {
        const float* S = p.S + (static_cast<size_t>(L.idx) * p.Hd * p.dv + b) * p.dk;
        s[n++] = {reinterpret_cast<const uint8_t*>(S), e - b, p.dk * 4};
        s[n++] = {L.w_outT + static_cast<size_t>(b) * rb, e - b, rb};
      }
      break;
    }
    case kPhAttOut: {
      split_range(p.Hq * p.D, cta, G, b, e);
      if (e > b) s[n++] = {L.w_outT + static_cast<size_t>(b) * rb, e - b, rb};
      break;
    }
    case kPhMlp: {
      split_range(p.F, cta, G, b, e);
      if (e > b) {
        s[n++] = {L.w_gate + static_cast<size_t>(b) * rb, e - b, rb};
        s[n++] = {L.w_up + static_cast<size_t>(b) * rb, e - b, rb};
        s[n++] = {L.w_downT + static_cast<size_t>(b) * rb, e - b, rb};
      }
      break;
    }
    default: {   // final: LM head rows (tied embedding)
      split_range(p.V, cta, G, b, e);
      if (e > b) s[n++] = {p.embed + static_cast<size_t>(b) * rb, e - b, rb};
      break;
    }
  }
  return n;
}

__device__ __forceinline__ int n_phases(const LayerW& L) { return L.kind == kDeltaNet ? 3 : 4; }
__device__ __forceinline__ int phase_id(const LayerW& L, int k) {
  if (L.kind == kDeltaNet) return k == 0 ? kPhIn : (k == 1 ? kPhMix : kPhMlp);
  return k == 0 ? kPhIn : (k == 1 ? kPhMix : (k == 2 ? kPhAttOut : kPhMlp));
}

// ------------------------------------------------------------------ producer
__device__ void producer_loop(const DecodeParams& p, Shared* sh, uint8_t* ring, int cta, int G) {
  const uint64_t pol = policy_evict_first();
  uint32_t n = 0;
  int last_in_slot[kSlots];
#pragma unroll
  for (int i = 0; i < kSlots; ++i) last_in_slot[i] = -1;
  volatile int* abort = &sh->abort_flag;
  bool ok = true;
  Seg segs[3];
  for (int l = 0; l <= p.n_layers && ok; ++l) {
    const bool final = (l == p.n_layers);
    const LayerW L = final ? LayerW{} : p.layers[l];
    const int nph = final ? 1 : n_phases(L);
    for (int k = 0; k < nph && ok; ++k) {
      const int ph = final ? static_cast<int>(kPhFinal) : phase_id(L, k);
      const int ns = phase_segments(p, L, ph, cta, G, segs);
      for (int si = 0; si < ns && ok; ++si) {
        const Seg sg = segs[si];
        const int rpc = kSlotBytes / sg.row_bytes;
        for (int r = 0; r < sg.rows; r += rpc) {
          const int nr = min(rpc, sg.rows - r);
          const uint32_t bytes = static_cast<uint32_t>(nr) * sg.row_bytes;
          const int slot = n % kSlots;
          if (n >= static_cast<uint32_t>(kSlots)) {
            if (!mbar_wait(&sh->empty[slot], ((n / kSlots) - 1) & 1, abort, kWaitLimitNs)) {
              if (!*abort) atomicOr(p.err, MK_DEVERR_PIPE_TIMEOUT);
              *abort = 1;
              ok = false;
              break;
            }
          }
          mbar_arrive_expect_tx(&sh->full[slot], bytes);
          bulk_g2s(ring + static_cast<size_t>(slot) * kSlotBytes, sg.src + static_cast<size_t>(r) * sg.row_bytes,
                   bytes, &sh->full[slot], pol);
          last_in_slot[slot] = static_cast<int>(n);
          ++n;
        }
      }
    }
  }
  // Let every issued copy land before this warp leaves (bounded).
  int never = 0;
  for (int s = 0; s < kSlots; ++s) {
    if (last_in_slot[s] >= 0)
      mbar_wait(&sh->full[s], (static_cast<uint32_t>(last_in_slot[s]) / kSlots) & 1, &never, kDrainLimitNs);
  }
}

// ------------------------------------------------------------------ consumer helpers
struct Cons {
  uint8_t* ring;
  Shared* sh;
  uint32_t n;      // next chunk index (same in all consumer threads)
  int tid, warp, lane;
};

__device__ __forceinline__ const uint8_t* acquire(Cons& c, int* err) {
  const int slot = c.n % kSlots;
  if (!mbar_wait(&c.sh->full[slot], (c.n / kSlots) & 1, &c.sh->abort_flag, kWaitLimitNs)) {
    if (c.lane == 0) {
      if (!c.sh->abort_flag) atomicOr(err, MK_DEVERR_PIPE_TIMEOUT);
      c.sh->abort_flag = 1;
    }
  }
  return c.ring + static_cast<size_t>(slot) * kSlotBytes;
}
__device__ __forceinline__ void release(Cons& c) {
  __syncwarp();
  if (c.lane == 0) mbar_arrive(&c.sh->empty[c.n % kSlots]);
  ++c.n;
}

// Grid-wide barrier among consumer thread groups of all CTAs. Returns false if this
// CTA must stop (own or remote failure); the result is the same in every consumer thread.
__device__ bool grid_barrier(const DecodeParams& p, Shared* sh, unsigned target) {
  cons_sync(kConsumerThreads);
  if (threadIdx.x == 0) {
    int stop = sh->abort_flag;
    if (!stop) {
      __threadfence();
      atomicAdd(p.bar, 1u);
      uint64_t t0 = 0;
      for (uint32_t it = 1;; ++it) {
        const unsigned v = ld_acquire(p.bar);
        if (static_cast<int>(v - target) >= 0) break;
        if ((it & 127) == 0) {
          if (ld_volatile(p.err) != 0 || sh->abort_flag) { stop = 1; break; }
          const uint64_t now = global_ns();
          if (t0 == 0) t0 = now;
          else if (now - t0 > kWaitLimitNs) {
            atomicOr(p.err, MK_DEVERR_BARRIER_TIMEOUT);
            stop = 1;
            break;
          }
        }
      }
      __threadfence();
    }
    if (stop) sh->abort_flag = 1;
    sh->decision = stop;
  }
  cons_sync(kConsumerThreads);
  return sh->decision == 0;
}

// Sum over all consumer threads; every consumer thread gets the total.
__device__ __forceinline__ float cons_sum(float v, Shared* sh, int warp, int lane) {
  v = warp_sum(v);
  cons_sync(kConsumerThreads);
  if (lane == 0) sh->red[warp] = v;
  cons_sync(kConsumerThreads);
  float t = (lane < kConsumerWarps) ? sh->red[lane] : 0.0f;
  return warp_sum(t);
}

// xs = h / sqrt(mean(h^2) + eps) * gamma   (fp32, kept on chip)
__device__ void rmsnorm_to_smem(const DecodeParams& p, const float* h, bool h_is_bf16_row, const uint8_t* bf_row,
                                const uint16_t* gamma, float* xs, Shared* sh, int tid, int warp, int lane) {
  float ss = 0.f;
  for (int c = tid; c < p.H; c += kConsumerThreads) {
    const float v = h_is_bf16_row ? bf16_to_f(reinterpret_cast<const uint16_t*>(bf_row)[c]) : __ldcg(h + c);
    ss = fmaf(v, v, ss);
  }
  ss = cons_sum(ss, sh, warp, lane);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(p.H) + p.eps);
  for (int c = tid; c < p.H; c += kConsumerThreads) {
    const float v = h_is_bf16_row ? bf16_to_f(reinterpret_cast<const uint16_t*>(bf_row)[c]) : __ldcg(h + c);
    xs[c] = v * inv * bf16_to_f(gamma[c]);
  }
  cons_sync(kConsumerThreads);
}

// Warp-per-row dot products of a chunk of bf16 rows with the fp32 vector xs;
// f(row, value) runs on lane 0.
template <class F>
__device__ __forceinline__ void gemv_chunk(const uint8_t* chunk, int nrows, int rb, const float* xs, int H,
                                           int warp, int lane, F&& f) {
  int r = warp;
  for (; r + kConsumerWarps < nrows; r += 2 * kConsumerWarps) {
    const uint8_t* r0 = chunk + static_cast<size_t>(r) * rb;
    const uint8_t* r1 = r0 + static_cast<size_t>(kConsumerWarps) * rb;
    float a0 = 0.f, a1 = 0.f;
    for (int c = lane * 8; c < H; c += 256) {
      const float4 xa = *reinterpret_cast<const float4*>(xs + c);
      const float4 xb = *reinterpret_cast<const float4*>(xs + c + 4);
      a0 = dot8_bf16_f32(*reinterpret_cast<const uint4*>(r0 + 2 * c), xa, xb, a0);
      a1 = dot8_bf16_f32(*reinterpret_cast<const uint4*>(r1 + 2 * c), xa, xb, a1);
    }
    a0 = warp_sum(a0);
    a1 = warp_sum(a1);
    if (lane == 0) { f(r, a0); f(r + kConsumerWarps, a1); }
  }
  for (; r < nrows; r += kConsumerWarps) {
    const uint8_t* r0 = chunk + static_cast<size_t>(r) * rb;
    float a0 = 0.f;
    for (int c = lane * 8; c < H; c += 256)
      a0 = dot8_bf16_f32(*reinterpret_cast<const uint4*>(r0 + 2 * c), *reinterpret_cast<const float4*>(xs + c),
                         *reinterpret_cast<const float4*>(xs + c + 4), a0);
    a0 = warp_sum(a0);
    if (lane == 0) f(r, a0);
  }
}

// Split-K accumulate: acc[out] += sum_r row_r[out] * coef[r] over a chunk of rows of
// length H (bf16). Thread tid owns float4 groups tid, tid + 256, ...
__device__ __forceinline__ void splitk_chunk(const uint8_t* chunk, int nrows, int rb, const float* coef, int H,
                                             int tid, float4* acc) {
  const int ng = H / 4;
  for (int r = 0; r < nrows; ++r) {
    const uint8_t* row = chunk + static_cast<size_t>(r) * rb;
    const float cf = coef[r];
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) {
        const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * g);
        acc[k].x = fmaf(bf16lo(w.x), cf, acc[k].x);
        acc[k].y = fmaf(bf16hi(w.x), cf, acc[k].y);
        acc[k].z = fmaf(bf16lo(w.y), cf, acc[k].z);
        acc[k].w = fmaf(bf16hi(w.y), cf, acc[k].w);
      }
    }
  }
}

// Residual update u: nxt += acc (+ cur from CTA 0); CTA G-1 zeroes the buffer that update u+1 adds into.
__device__ __forceinline__ void residual_epilogue(const DecodeParams& p, int u, bool has_rows, const float4* acc,
                                                  int cta, int G, int tid) {
  const int H = p.H;
  float* cur = p.hbuf + static_cast<size_t>(u % 3) * H;
  float* nxt = p.hbuf + static_cast<size_t>((u + 1) % 3) * H;
  float* third = p.hbuf + static_cast<size_t>((u + 2) % 3) * H;
  const int ng = H / 4;
  if (has_rows || cta == 0) {
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) {
        float4 a = acc[k];
        if (cta == 0) {
          const float4 c = __ldcg(reinterpret_cast<const float4*>(cur) + g);
          a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
        }
        atomicAdd(reinterpret_cast<float4*>(nxt) + g, a);
      }
    }
  }
  if (cta == G - 1) {
    for (int g = tid; g < ng; g += kConsumerThreads)
      __stcg(reinterpret_cast<float4*>(third) + g, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kThreads, 1) mk_decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  Shared* sh = reinterpret_cast<Shared*>(smem + static_cast<size_t>(kSlots) * kSlotBytes);
  float* fs = reinterpret_cast<float*>(sh + 1);                          // scratch [kScratchFloats]
  float* xs = fs + kScratchFloats;                                       // normed input [H] fp32

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, G = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], kConsumerWarps);
    }
    fence_barrier_init();
    sh->abort_flag = 0;
    sh->decision = 0;
    const int e = ld_volatile(p.err);
    const int pos = ld_volatile(p.pos);
    const int tok = ld_volatile(p.in_token);
    sh->pos = pos;
    sh->tok = tok;
    int bad = (e != 0);
    if (!bad && (tok < 0 || tok >= p.V)) {
      bad = 1;
      if (cta == 0) atomicOr(p.err, MK_DEVERR_BAD_TOKEN);
    }
    if (!bad && (pos < 0 || pos >= p.max_ctx)) {
      bad = 1;
      if (cta == 0) atomicOr(p.err, MK_DEVERR_CAPACITY);
    }
    if (!bad && p.gate_n && p.gate_i > ld_volatile(p.gate_n)) bad = 1;   // skipped replay step
    sh->bad = bad;
  }
  __syncthreads();
  if (sh->bad) return;

  if (warp == kConsumerWarps) {
    if (lane == 0) producer_loop(p, sh, ring, cta, G);
    return;
  }

  // ---------------- consumers ----------------
  Cons cs{ring, sh, 0u, tid, warp, lane};
  const int pos = sh->pos;
  const int tok = sh->tok;
  const uint8_t* emb_row = p.embed + static_cast<size_t>(tok) * p.row_bytes;
  const int rb = p.row_bytes;
  unsigned nbar = 0;
  int u = 0;                    // residual update counter
  Seg segs[3];

  for (int l = 0; l < p.n_layers; ++l) {
    const LayerW L = p.layers[l];
    const int nph = n_phases(L);
    for (int k = 0; k < nph; ++k) {
      const int ph = phase_id(L, k);
      if (l > 0 || k > 0) {
        if (!grid_barrier(p, sh, ++nbar * static_cast<unsigned>(G))) return;
      }
      const int ns = phase_segments(p, L, ph, cta, G, segs);

      if (ph == kPhIn) {
        // ---- pre-mixer RMSNorm + input projection ----
        if (l == 0) {
          rmsnorm_to_smem(p, nullptr, true, emb_row, L.norm1, xs, sh, tid, warp, lane);
          if (cta == 0) {     // residual stream starts as the embedding row
            for (int c = tid; c < p.H; c += kConsumerThreads) {
              __stcg(p.hbuf + c, bf16_to_f(reinterpret_cast<const uint16_t*>(emb_row)[c]));
              __stcg(p.hbuf + p.H + c, 0.f);
            }
          }
        } else {
          rmsnorm_to_smem(p, p.hbuf + static_cast<size_t>(u % 3) * p.H, false, nullptr, L.norm1, xs, sh, tid,
                          warp, lane);
        }
        int b = 0, e = 0;
        const int rows = (L.kind == kDeltaNet) ? (p.C + 2 * p.Hd) : p.at_in_rows;
        split_range(rows, cta, G, b, e);
        if (ns) {
          const Seg sg = segs[0];
          const int rpc = kSlotBytes / sg.row_bytes;
          float* ringc = p.conv_ring + static_cast<size_t>(L.idx) * p.convw * p.C +
                         static_cast<size_t>(pos % p.convw) * p.C;
          for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
            const int nr = min(rpc, sg.rows - r0);
            const uint8_t* ch = acquire(cs, p.err);
            const int base = b + r0;
            if (L.kind == kDeltaNet) {
              gemv_chunk(ch, nr, rb, xs, p.H, warp, lane, [&](int r, float v) {
                const int row = base + r;
                if (row < p.C) __stcg(ringc + row, v);
                else __stcg(p.z + (row - p.C), v);
              });
            } else {
              gemv_chunk(ch, nr, rb, xs, p.H, warp, lane, [&](int r, float v) { __stcg(p.z + base + r, v); });
            }
            release(cs);
          }
        }
      } else if (ph == kPhMix && L.kind == kDeltaNet) {
        // ---- conv + SiLU + L2 norm + gates, gated delta rule on this CTA's rows of S, out-proj split-K ----
        int g0 = 0, g1 = 0;
        split_range(p.Hd * p.dv, cta, G, g0, g1);
        const int nrows = g1 - g0;
        float4 acc[kMaxGroups];
#pragma unroll
        for (int q = 0; q < kMaxGroups; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (nrows > 0) {
          const int h0 = g0 / p.dv, h1 = (g1 - 1) / p.dv;
          const int nh = h1 - h0 + 1;
          // scratch layout: qk[nh][2][dk] | ab[nh][2] | vv[nrows] | oc[nrows]
          float* qk = fs;
          float* ab = qk + nh * 2 * p.dk;
          float* vv = ab + 2 * nh;
          float* oc = vv + nrows;
          const float* ringl = p.conv_ring + static_cast<size_t>(L.idx) * p.convw * p.C;
          const uint16_t* taps = L.conv;
          auto conv_at = [&](int ch) -> float {
            float y = 0.f;
            for (int j = 0; j < p.convw; ++j) {
              int src = pos - (p.convw - 1) + j;
              int slot = ((src % p.convw) + p.convw) % p.convw;
              y = fmaf(bf16_to_f(taps[static_cast<size_t>(ch) * p.convw + j]),
                       __ldcg(ringl + static_cast<size_t>(slot) * p.C + ch), y);
            }
            return siluf_(y);
          };
          // q and k vectors: one warp per (head, q|k) vector, with its L2 norm
          for (int vec = warp; vec < 2 * nh; vec += kConsumerWarps) {
            const int hh = h0 + (vec >> 1);
            const int isk = vec & 1;
            const int chb = isk ? (p.Hd * p.dk + hh * p.dk) : (hh * p.dk);
            float* dst = qk + vec * p.dk;
            float ss = 0.f;
            for (int i = lane; i < p.dk; i += 32) {
              const float y = conv_at(chb + i);
              dst[i] = y;
              ss = fmaf(y, y, ss);
            }
            ss = warp_sum(ss);
            const float inv = 1.0f / sqrtf(ss + 1e-6f);
            __syncwarp();
            for (int i = lane; i < p.dk; i += 32) dst[i] *= inv;
          }
          for (int i = tid; i < nh; i += kConsumerThreads) {
            const float al = __ldcg(p.z + h0 + i);
            const float be = __ldcg(p.z + p.Hd + h0 + i);
            ab[2 * i] = sigmoidf_(-al);        // exp(-softplus(alpha))
            ab[2 * i + 1] = sigmoidf_(be);
          }
          for (int r = tid; r < nrows; r += kConsumerThreads) {
            const int g = g0 + r;
            vv[r] = conv_at(2 * p.Hd * p.dk + g);   // v channel of (head g/dv, row g%dv)
          }
          cons_sync(kConsumerThreads);
          // S rows (fp32) through the ring
          {
            const Seg sg = segs[0];
            const int rpc = kSlotBytes / sg.row_bytes;
            const int vpl = p.dk / 32;
            for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
              const int nr = min(rpc, sg.rows - r0);
              const float* ch = reinterpret_cast<const float*>(acquire(cs, p.err));
              for (int r = warp; r < nr; r += kConsumerWarps) {
                const int lr = r0 + r;
                const int g = g0 + lr;
                const int hl = g / p.dv - h0;
                const float a = ab[2 * hl], bb = ab[2 * hl + 1];
                const float* qv = qk + (2 * hl) * p.dk;
                const float* kv = qk + (2 * hl + 1) * p.dk;
                const float* srow = ch + static_cast<size_t>(r) * p.dk;
                float s[8];
                float ukk = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  if (q < vpl) {
                    s[q] = a * srow[lane + 32 * q];
                    ukk = fmaf(s[q], kv[lane + 32 * q], ukk);
                  }
                }
                ukk = warp_sum(ukk);
                const float coef = bb * (vv[lr] - ukk);
                float o = 0.f;
                float* sg_out = p.S + (static_cast<size_t>(L.idx) * p.Hd * p.dv + g) * p.dk;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  if (q < vpl) {
                    s[q] = fmaf(coef, kv[lane + 32 * q], s[q]);
                    o = fmaf(s[q], qv[lane + 32 * q], o);
                    __stcg(sg_out + lane + 32 * q, s[q]);
                  }
                }
                o = warp_sum(o);
                if (lane == 0) oc[lr] = o;
              }
              release(cs);
            }
          }
          cons_sync(kConsumerThreads);
          // out-projection, split over this CTA's value rows
          {
            const Seg sg = segs[1];
            const int rpc = kSlotBytes / sg.row_bytes;
            for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
              const int nr = min(rpc, sg.rows - r0);
              const uint8_t* ch = acquire(cs, p.err);
              splitk_chunk(ch, nr, rb, oc + r0, p.H, tid, acc);
              release(cs);
            }
          }
        }
        residual_epilogue(p, u, nrows > 0, acc, cta, G, tid);
        ++u;
      } else if (ph == kPhMix) {
        // ---- attention: RoPE, KV append, split-K partial softmax over the cache ----
        const int n = pos + 1;
        int CH, nsplit;
        attn_split(n, G, p.Hkv, p.max_splits, CH, nsplit);
        const int grp = p.Hq / p.Hkv;
        const int D = p.D, half = D / 2;
        const float scale = 1.0f / sqrtf(static_cast<float>(D));
        const int qoff = 0;
        const int koff = p.Hq * D * (p.gated ? 2 : 1);
        const int voff = koff + p.Hkv * D;
        float* qs = fs;                       // [grp][D]
        float* sc = qs + grp * D;             // [grp][kAttnSub]
        float* mlc = sc + grp * kAttnSub;     // [grp][3]: m, l, corr
        const size_t cache_base = static_cast<size_t>(L.idx) * p.Hkv * p.max_ctx * D;
        const int units = p.Hkv * nsplit;
        for (int un = cta; un < units; un += G) {
          const int g = un % p.Hkv, j = un / p.Hkv;
          const int p0 = j * CH, p1 = min(n, p0 + CH);
          uint16_t* Kg = p.kc + cache_base + static_cast<size_t>(g) * p.max_ctx * D;
          uint16_t* Vg = p.vc + cache_base + static_cast<size_t>(g) * p.max_ctx * D;
          for (int idx = tid; idx < grp * half; idx += kConsumerThreads) {
            const int t = idx / half, i = idx % half;
            const int hq = g * grp + t;
            double sn, cn;
            sincos(static_cast<double>(pos) * p.inv_freq[i], &sn, &cn);
            const float c = static_cast<float>(cn), s = static_cast<float>(sn);
            const float x1 = __ldcg(p.z + qoff + hq * D + i), x2 = __ldcg(p.z + qoff + hq * D + i + half);
            qs[t * D + i] = (x1 * c - x2 * s) * scale;
            qs[t * D + i + half] = (x1 * s + x2 * c) * scale;
          }
          if (p1 == n) {   // this unit holds the current position: append k, v (bf16)
            for (int i = tid; i < half; i += kConsumerThreads) {
              double sn, cn;
              sincos(static_cast<double>(pos) * p.inv_freq[i], &sn, &cn);
              const float c = static_cast<float>(cn), s = static_cast<float>(sn);
              const float x1 = __ldcg(p.z + koff + g * D + i), x2 = __ldcg(p.z + koff + g * D + i + half);
              Kg[static_cast<size_t>(pos) * D + i] = f_to_bf16(x1 * c - x2 * s);
              Kg[static_cast<size_t>(pos) * D + i + half] = f_to_bf16(x1 * s + x2 * c);
            }
            for (int d = tid; d < D; d += kConsumerThreads)
              Vg[static_cast<size_t>(pos) * D + d] = f_to_bf16(__ldcg(p.z + voff + g * D + d));
          }
          if (tid < grp) {
            mlc[3 * tid] = -INFINITY;
            mlc[3 * tid + 1] = 0.f;
            mlc[3 * tid + 2] = 0.f;
          }
          float oacc[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) oacc[t] = 0.f;
          cons_sync(kConsumerThreads);
          const int dpl = D / 32;      // dims per lane (2..8)
          for (int sb = p0; sb < p1; sb += kAttnSub) {
            const int np = min(kAttnSub, p1 - sb);
            for (int pp = warp; pp < np; pp += kConsumerWarps) {
              const uint16_t* krow = Kg + static_cast<size_t>(sb + pp) * D + lane * dpl;
              float kf[8];
              if (dpl == 8) {
                const uint4 kw = __ldcg(reinterpret_cast<const uint4*>(krow));
                kf[0] = bf16lo(kw.x); kf[1] = bf16hi(kw.x); kf[2] = bf16lo(kw.y); kf[3] = bf16hi(kw.y);
                kf[4] = bf16lo(kw.z); kf[5] = bf16hi(kw.z); kf[6] = bf16lo(kw.w); kf[7] = bf16hi(kw.w);
              } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) kf[q] = (q < dpl) ? bf16_to_f(__ldcg(krow + q)) : 0.f;
              }
              for (int t = 0; t < grp; ++t) {
                const float* qv = qs + t * D + lane * dpl;
                float d0 = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  if (q < dpl) d0 = fmaf(qv[q], kf[q], d0);
                d0 = warp_sum(d0);
                if (lane == 0) sc[t * kAttnSub + pp] = d0;
              }
            }
            cons_sync(kConsumerThreads);
            if (warp < grp) {
              const int t = warp;
              float mx = -INFINITY;
              for (int pp = lane; pp < np; pp += 32) mx = fmaxf(mx, sc[t * kAttnSub + pp]);
              mx = warp_max(mx);
              const float m_old = mlc[3 * t];
              const float m_new = fmaxf(m_old, mx);
              float ls = 0.f;
              for (int pp = lane; pp < np; pp += 32) {
                const float e = expf(sc[t * kAttnSub + pp] - m_new);
                sc[t * kAttnSub + pp] = e;
                ls += e;
              }
              ls = warp_sum(ls);
              __syncwarp();
              if (lane == 0) {
                const float corr = expf(m_old - m_new);
                mlc[3 * t] = m_new;
                mlc[3 * t + 1] = mlc[3 * t + 1] * corr + ls;
                mlc[3 * t + 2] = corr;
              }
            }
            cons_sync(kConsumerThreads);
            if (tid < D) {
              float vsum[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) vsum[t] = 0.f;
              for (int pp = 0; pp < np; ++pp) {
                const float vv = bf16_to_f(__ldcg(Vg + static_cast<size_t>(sb + pp) * D + tid));
#pragma unroll
                for (int t = 0; t < 8; ++t)
                  if (t < grp) vsum[t] = fmaf(sc[t * kAttnSub + pp], vv, vsum[t]);
              }
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (t < grp) oacc[t] = oacc[t] * mlc[3 * t + 2] + vsum[t];
            }
            cons_sync(kConsumerThreads);
          }
          // partials: [hq][split][D + 2] = acc..., m, l
          if (tid < D) {
            for (int t = 0; t < grp; ++t) {
              const int hq = g * grp + t;
              float* dst = p.part + (static_cast<size_t>(hq) * p.max_splits + j) * (D + 2);
              __stcg(dst + tid, oacc[t]);
            }
          }
          if (tid < grp) {
            const int hq = g * grp + tid;
            float* dst = p.part + (static_cast<size_t>(hq) * p.max_splits + j) * (D + 2);
            __stcg(dst + D, mlc[3 * tid]);
            __stcg(dst + D + 1, mlc[3 * tid + 1]);
          }
          cons_sync(kConsumerThreads);
        }
      } else if (ph == kPhAttOut) {
        // ---- combine split-K partials for this CTA's output columns, gate, out-proj split-K ----
        const int n = pos + 1;
        int CH, nsplit;
        attn_split(n, G, p.Hkv, p.max_splits, CH, nsplit);
        int c0 = 0, c1 = 0;
        split_range(p.Hq * p.D, cta, G, c0, c1);
        const int ncol = c1 - c0;
        float4 acc[kMaxGroups];
#pragma unroll
        for (int q = 0; q < kMaxGroups; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        float* oc = fs;
        for (int cc = tid; cc < ncol; cc += kConsumerThreads) {
          const int col = c0 + cc;
          const int hq = col / p.D, d = col % p.D;
          const float* base = p.part + static_cast<size_t>(hq) * p.max_splits * (p.D + 2);
          float M = -INFINITY;
          for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(base + static_cast<size_t>(j) * (p.D + 2) + p.D));
          float Ls = 0.f, O = 0.f;
          for (int j = 0; j < nsplit; ++j) {
            const float* pj = base + static_cast<size_t>(j) * (p.D + 2);
            const float w = expf(__ldcg(pj + p.D) - M);
            Ls = fmaf(__ldcg(pj + p.D + 1), w, Ls);
            O = fmaf(__ldcg(pj + d), w, O);
          }
          float o = O / Ls;
          if (p.gated) o *= sigmoidf_(__ldcg(p.z + p.Hq * p.D + col));
          oc[cc] = o;
        }
        cons_sync(kConsumerThreads);
        if (ns) {
          const Seg sg = segs[0];
          const int rpc = kSlotBytes / sg.row_bytes;
          for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
            const int nr = min(rpc, sg.rows - r0);
            const uint8_t* ch = acquire(cs, p.err);
            splitk_chunk(ch, nr, rb, oc + r0, p.H, tid, acc);
            release(cs);
          }
        }
        residual_epilogue(p, u, ncol > 0, acc, cta, G, tid);
        ++u;
      } else {
        // ---- pre-MLP RMSNorm, SwiGLU gate/up for this CTA's intermediate rows, down split-K ----
        rmsnorm_to_smem(p, p.hbuf + static_cast<size_t>(u % 3) * p.H, false, nullptr, L.norm2, xs, sh, tid, warp,
                        lane);
        int j0 = 0, j1 = 0;
        split_range(p.F, cta, G, j0, j1);
        const int nj = j1 - j0;
        float4 acc[kMaxGroups];
#pragma unroll
        for (int q = 0; q < kMaxGroups; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        float* gs = fs;
        float* act = fs + nj;
        if (ns) {
          for (int si = 0; si < 2; ++si) {
            const Seg sg = segs[si];
            const int rpc = kSlotBytes / sg.row_bytes;
            for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
              const int nr = min(rpc, sg.rows - r0);
              const uint8_t* ch = acquire(cs, p.err);
              if (si == 0) {
                gemv_chunk(ch, nr, rb, xs, p.H, warp, lane, [&](int r, float v) { gs[r0 + r] = v; });
              } else {
                gemv_chunk(ch, nr, rb, xs, p.H, warp, lane,
                           [&](int r, float v) { act[r0 + r] = siluf_(gs[r0 + r]) * v; });
              }
              release(cs);
            }
            cons_sync(kConsumerThreads);
          }
          const Seg sg = segs[2];
          const int rpc = kSlotBytes / sg.row_bytes;
          for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
            const int nr = min(rpc, sg.rows - r0);
            const uint8_t* ch = acquire(cs, p.err);
            splitk_chunk(ch, nr, rb, act + r0, p.H, tid, acc);
            release(cs);
          }
        }
        residual_epilogue(p, u, nj > 0, acc, cta, G, tid);
        ++u;
      }
    }
  }

  // ---------------- final norm, tied LM head, argmax ----------------
  if (!grid_barrier(p, sh, ++nbar * static_cast<unsigned>(G))) return;
  rmsnorm_to_smem(p, p.hbuf + static_cast<size_t>(u % 3) * p.H, false, nullptr, p.norm_f, xs, sh, tid, warp, lane);
  {
    const LayerW dummy{};
    const int ns = phase_segments(p, dummy, kPhFinal, cta, G, segs);
    int v0 = 0, v1 = 0;
    split_range(p.V, cta, G, v0, v1);
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
    if (ns) {
      const Seg sg = segs[0];
      const int rpc = kSlotBytes / sg.row_bytes;
      for (int r0 = 0; r0 < sg.rows; r0 += rpc) {
        const int nr = min(rpc, sg.rows - r0);
        const uint8_t* ch = acquire(cs, p.err);
        gemv_chunk(ch, nr, rb, xs, p.H, warp, lane, [&](int r, float v) {
          const int idx = v0 + r0 + r;
          if (p.logits) __stcg(p.logits + idx, v);
          if (v > bv || (v == bv && idx < bi)) { bv = v; bi = idx; }
        });
        release(cs);
      }
    }
    if (lane == 0) {
      sh->best_v[warp] = bv;
      sh->best_i[warp] = bi;
    }
    cons_sync(kConsumerThreads);
    if (tid == 0) {
      float cv = -INFINITY;
      int ci = 0x7FFFFFFF;
      for (int w = 0; w < kConsumerWarps; ++w) {
        if (sh->best_i[w] == 0x7FFFFFFF) continue;
        if (sh->best_v[w] > cv || (sh->best_v[w] == cv && sh->best_i[w] < ci)) {
          cv = sh->best_v[w];
          ci = sh->best_i[w];
        }
      }
      if (ci != 0x7FFFFFFF) atomicMax(p.amax, pack_argmax(cv, ci));
      __threadfence();
      const unsigned prev = atomicAdd(p.done, 1u);
      if (prev == static_cast<unsigned>(G - 1)) {
        __threadfence();
        const unsigned long long best = atomicAdd(p.amax, 0ull);
        *p.out_token = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best & 0xFFFFFFFFull));
        *p.pos = pos + 1;
        *p.amax = 0ull;
        *p.done = 0u;
        *p.bar = 0u;
        __threadfence();
      }
    }
  }
}

size_t decode_smem_bytes(int H) {
  return static_cast<size_t>(kSlots) * kSlotBytes + sizeof(Shared) + kScratchFloats * sizeof(float) +
         static_cast<size_t>(H) * 4;
}

int decode_max_splits(int grid, int hkv) {
  int per = grid / hkv;
  return per < 1 ? 1 : per;
}

cudaError_t launch_decode(const DecodeParams& p, int grid, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(p.H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(mk_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem > 232448 ? 232448 : 232448));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mk_decode_kernel, p);
}

int decode_grid_for_device(int device, int* grid_out) {
  int sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return -1;
  *grid_out = sms;
  return 0;
}

}  // namespace mk
