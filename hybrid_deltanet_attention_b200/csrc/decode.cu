// Persistent decode megakernel: one launch runs every layer of one batch-1 forward step.
//
// Design (the Hacker News post on the fused Qwen3.5-0.8B kernel, design bullets, is
// the prior art: one launch per token, persistent blocks on every SM, a grid-wide
// barrier instead of kernel boundaries; re-done here for sm_100a):
//  * grid = one CTA per SM (cooperative launch, so all CTAs are co-resident);
//  * each CTA owns a fixed contiguous slice of every weight matrix, of the DeltaNet
//    state rows, and of the KV cache positions of its attention split. Its slice
//    bounds are computed once per launch into shared memory. A producer lane streams
//    that whole per-step sequence through a 3 x 64 KB shared-memory ring with
//    cp.async.bulk (no multicast), independent of the grid barriers; its per-chunk
//    work is a handful of instructions so it never limits the stream;
//  * 8 consumer warps do the arithmetic in fp32 from shared memory; activations never
//    leave the chip except the small vectors exchanged between phases (L2);
//  * out-projections and the MLP down-projection are split over their input dim
//    (split-K) and added to the residual with vector reductions, so a DeltaNet layer
//    needs 3 grid barriers and an attention layer 4;
//  * every wait (grid barrier, pipeline slot) has a time limit; on expiry the kernel
//    latches a bit in the device error word and every CTA returns.
#include <cuda_fp16.h>

#include "dev.cuh"
#include "mk_internal.h"
#include "../../include/mk.h"

namespace mk {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: a healthy wait takes microseconds
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 200 ms for in-flight copies to land
constexpr int kMaxConv = 4;          // causal conv width limit (the configs use 4)
constexpr int kConvItems = 3;        // conv items per consumer thread in the DeltaNet prologue
constexpr int kNoSplit = 0x7FFFFFFF;
constexpr int kMaxHead = 256;        // largest attention head dim

// Per-CTA slice bounds, computed once per launch by thread 0.
struct Ranges {
  int in_dn_b, in_dn_e;   // DeltaNet in-projection rows
  int in_at_b, in_at_e;   // attention in-projection rows
  int dn_b, dn_e;         // DeltaNet state rows (head*dv + i) and out-projection columns
  int col_b, col_e;       // attention output columns (out-projection split-K)
  int f_b, f_e;           // MLP intermediate rows
  int v_b, v_e;           // LM-head rows
  int h_b, h_e;           // output rows of the out- and down-projections (Q4 weights)
  int au_valid, au_g, au_j, au_p0, au_p1, au_q1;   // attention split unit
  int nsplit;
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
  float rope_c[kMaxHead / 2];   // cos / sin of pos * inv_freq_i for this launch's position
  float rope_s[kMaxHead / 2];
  float best_v[kConsumerWarps];
  int best_i[kConsumerWarps];
  Ranges rg;
};

// Shared-memory copy of the layer table (16-byte multiple): every layer's entry, copied at
// launch start, when the budget allows (p.ltab_full); otherwise two slots, layer l + 1's
// entry fetched into slot (l + 1) & 1 while layer l runs.
__host__ __device__ constexpr size_t layer_table_bytes(int entries) {
  return (static_cast<size_t>(entries) * sizeof(LayerW) + 15) / 16 * 16;
}
static_assert(sizeof(LayerW) % 4 == 0, "layer entries are copied in 32-bit words");
static_assert(sizeof(Shared) % 16 == 0, "the layer table and xs follow Shared 16-byte aligned");

__device__ __forceinline__ void split_range(int n, int c, int G, int& b, int& e) {
  b = static_cast<int>((static_cast<long long>(n) * c) / G);
  e = static_cast<int>((static_cast<long long>(n) * (c + 1)) / G);
}

// Split of the n = pos + 1 cached positions into chunks of CH positions so that
// Hkv * nsplit <= grid (every CTA owns at most one (kv head, chunk) unit).
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

__device__ void compute_ranges(const DecodeParams& p, int cta, int G, int pos, Ranges& r) {
  split_range(p.C + 2 * p.Hd, cta, G, r.in_dn_b, r.in_dn_e);
  split_range(p.at_in_rows, cta, G, r.in_at_b, r.in_at_e);
  split_range(p.Hd * p.dv, cta, G, r.dn_b, r.dn_e);
  split_range(p.Hq * p.D, cta, G, r.col_b, r.col_e);
  split_range(p.F, cta, G, r.f_b, r.f_e);
  split_range(p.V, cta, G, r.v_b, r.v_e);
  split_range(p.H, cta, G, r.h_b, r.h_e);
  const int n = pos + 1;
  int CH = 1, nsplit = 1;
  if (p.Hkv > 0) attn_split(n, G, p.Hkv, p.max_splits, CH, nsplit);
  r.nsplit = nsplit;
  r.au_valid = (p.Hkv > 0 && cta < p.Hkv * nsplit) ? 1 : 0;
  if (r.au_valid) {
    r.au_g = cta % p.Hkv;
    r.au_j = cta / p.Hkv;
    r.au_p0 = r.au_j * CH;
    r.au_p1 = min(n, r.au_p0 + CH);
    r.au_q1 = min(r.au_p1, pos);
  } else {
    r.au_g = r.au_j = r.au_p0 = r.au_p1 = r.au_q1 = 0;
  }
}

// Diagnostics (off unless p.trace is set): CTA 0 stamps its SM cycle counter. Entries
// below kTraceChunks: phase boundaries; from kTraceChunks: chunk n issued (4n), warp 0
// starts waiting for it (4n+1), has it (4n+2), is done with it (4n+3).
constexpr int kTraceChunks = 512;
// From kTraceGrid: every CTA stamps %globaltimer (ns) when it arrives at grid barrier k
// (entry kTraceGrid + 2 (k G + cta)) and when it leaves it (the next entry).
constexpr int kTraceGrid = 16384;
__device__ __forceinline__ void trace_at(const DecodeParams& p, int idx) {
  if (p.trace && blockIdx.x == 0 && idx < p.trace_cap && idx < kTraceGrid) p.trace[idx] = clock64();
}
__device__ __forceinline__ void trace_grid(const DecodeParams& p, unsigned k, int leave) {
  if (!p.trace) return;
  const long long ix = kTraceGrid + 2ll * (static_cast<long long>(k) * gridDim.x + blockIdx.x) + leave;
  if (ix < p.trace_cap) p.trace[ix] = global_ns();
}

// ------------------------------------------------------------------ producer
// Segment s of layer l in stream order (weights, DeltaNet state rows, KV sub-blocks);
// returns false past the end of the layer. The final "layer" p.n_layers is the LM head.
template <bool Q4>
__device__ __forceinline__ bool layer_segment(const DecodeParams& p, const Ranges& r, const LayerW& L, int l, int s,
                                              const uint8_t*& src, int& rows, int& rb) {
  const int wrb = p.row_bytes;
  if constexpr (Q4) {
    // order: in-proj | (S rows or KV sub-blocks...) | W_out rows | gate | up | W_down rows
    if (l == p.n_layers) {
      if (s > 0) return false;
      src = p.embed + static_cast<size_t>(r.v_b) * wrb;
      rows = r.v_e - r.v_b;
      rb = wrb;
      return true;
    }
    const bool dn = L.kind == kDeltaNet;
    const int nkv = (!dn && r.au_valid && r.au_q1 > r.au_p0) ? 2 * ((r.au_q1 - r.au_p0 + kAttnSub - 1) / kAttnSub) : 0;
    if (s == 0) {
      const int b = dn ? r.in_dn_b : r.in_at_b, e = dn ? r.in_dn_e : r.in_at_e;
      rb = dn ? wrb + 16 : wrb;
      src = L.w_in + static_cast<size_t>(b) * rb;
      rows = e - b;
      return true;
    }
    s -= 1;
    const int nmix = dn ? 1 : nkv;
    if (s < nmix) {
      if (dn) {
        src = reinterpret_cast<const uint8_t*>(p.S + (static_cast<size_t>(L.idx) * p.Hd * p.dv + r.dn_b) * p.dk);
        rows = r.dn_e - r.dn_b;
        rb = p.dk * 4;
      } else {
        const int sb = r.au_p0 + (s >> 1) * kAttnSub;
        src = reinterpret_cast<const uint8_t*>((s & 1) ? p.vc : p.kc) +
              ((static_cast<size_t>(L.idx) * p.Hkv + r.au_g) * p.max_ctx + sb) * p.kv_rb;
        rows = min(kAttnSub, r.au_q1 - sb);
        rb = p.kv_rb;
      }
      return true;
    }
    s -= nmix;
    if (s == 0) {
      rb = dn ? p.rb_dn_out : p.rb_at_out;
      src = L.w_out_q4 + static_cast<size_t>(r.h_b) * rb;
      rows = r.h_e - r.h_b;
      return true;
    }
    if (s == 1 || s == 2) {
      src = (s == 1 ? L.w_gate : L.w_up) + static_cast<size_t>(r.f_b) * wrb;
      rows = r.f_e - r.f_b;
      rb = wrb;
      return true;
    }
    if (s == 3) {
      rb = p.rb_ffn;
      src = L.w_down_q4 + static_cast<size_t>(r.h_b) * rb;
      rows = r.h_e - r.h_b;
      return true;
    }
    return false;
  }
  if (l == p.n_layers) {
    if (s > 0) return false;
    src = p.embed + static_cast<size_t>(r.v_b) * wrb;
    rows = r.v_e - r.v_b;
    rb = wrb;
    return true;
  }
  const int nkv = (L.kind == kAttention && r.au_valid && r.au_q1 > r.au_p0)
                      ? 2 * ((r.au_q1 - r.au_p0 + kAttnSub - 1) / kAttnSub) : 0;
  // order: in-proj | (S rows, out^T rows) or (KV sub-blocks..., out^T rows) | gate | up | down^T
  if (s == 0) {
    const int b = L.kind == kDeltaNet ? r.in_dn_b : r.in_at_b;
    const int e = L.kind == kDeltaNet ? r.in_dn_e : r.in_at_e;
    rb = L.kind == kDeltaNet ? wrb + 16 : wrb;     // DeltaNet rows carry their conv taps
    src = L.w_in + static_cast<size_t>(b) * rb;
    rows = e - b;
    return true;
  }
  s -= 1;
  if (L.kind == kDeltaNet) {
    if (s == 0) {
      src = reinterpret_cast<const uint8_t*>(p.S + (static_cast<size_t>(L.idx) * p.Hd * p.dv + r.dn_b) * p.dk);
      rows = r.dn_e - r.dn_b;
      rb = p.dk * 4;
      return true;
    }
    if (s == 1) {
      src = L.w_outT + static_cast<size_t>(r.dn_b) * wrb;
      rows = r.dn_e - r.dn_b;
      rb = wrb;
      return true;
    }
    s -= 2;
  } else {
    if (s < nkv) {
      const int sb = r.au_p0 + (s >> 1) * kAttnSub;
      src = reinterpret_cast<const uint8_t*>((s & 1) ? p.vc : p.kc) +
            ((static_cast<size_t>(L.idx) * p.Hkv + r.au_g) * p.max_ctx + sb) * p.kv_rb;
      rows = min(kAttnSub, r.au_q1 - sb);
      rb = p.kv_rb;
      return true;
    }
    s -= nkv;
    if (s == 0) {
      src = L.w_outT + static_cast<size_t>(r.col_b) * wrb;
      rows = r.col_e - r.col_b;
      rb = wrb;
      return true;
    }
    s -= 1;
  }
  if (s < 3) {
    const uint8_t* m = s == 0 ? L.w_gate : (s == 1 ? L.w_up : L.w_downT);
    src = m + static_cast<size_t>(r.f_b) * wrb;
    rows = r.f_e - r.f_b;
    rb = wrb;
    return true;
  }
  return false;
}

// One lane streams the CTA's chunks into the shared-memory ring: every segment that
// seg(p, r, L, l, s, src, rows, rb) yields for layers l = 0 .. n_layers (the last one the LM
// head), in chunks of whole rows of up to kSlotBytes. Consumers take the chunks in the same
// order. The layer table entry of layer l + 1 is loaded while layer l streams.
template <int NS, typename Seg>
__device__ void producer_walk(const DecodeParams& p, Shared* sh, uint8_t* ring, Seg&& seg) {
  const uint64_t pol = policy_evict_first();
  const Ranges r = sh->rg;
  volatile int* abort = &sh->abort_flag;
  uint32_t n = 0;
  bool ok = true;
  LayerW L = p.layers[0];
  for (int l = 0; l <= p.n_layers && ok; ++l) {
    const LayerW Lnext = (l + 1 < p.n_layers) ? p.layers[l + 1] : L;   // load ahead of use
    const uint8_t* src;
    int rows, rb;
    for (int s = 0; ok && seg(p, r, L, l, s, src, rows, rb); ++s) {
      const int rpc = kSlotBytes / rb;
      for (int r0 = 0; r0 < rows; r0 += rpc) {
        const uint32_t bytes = static_cast<uint32_t>(min(rpc, rows - r0)) * rb;
        const int slot = n % NS;
        if (n >= static_cast<uint32_t>(NS)) {
          if (!mbar_wait(&sh->empty[slot], ((n / NS) - 1) & 1, abort, kWaitLimitNs)) {
            if (!*abort) atomicOr(p.err, MK_DEVERR_PIPE_TIMEOUT);
            *abort = 1;
            ok = false;
            break;
          }
        }
        mbar_arrive_expect_tx(&sh->full[slot], bytes);
        bulk_g2s(ring + static_cast<size_t>(slot) * kSlotBytes, src + static_cast<size_t>(r0) * rb, bytes,
                 &sh->full[slot], pol);
        trace_at(p, kTraceChunks + 4 * static_cast<int>(n));
        ++n;
      }
    }
    L = Lnext;
  }
  // Let every issued copy land before this lane leaves (bounded): the last chunk
  // issued to each slot is one of the last NS chunks.
  int never = 0;
  for (uint32_t m = (n > static_cast<uint32_t>(NS) ? n - NS : 0); m < n; ++m)
    mbar_wait(&sh->full[m % NS], (m / NS) & 1, &never, kDrainLimitNs);
}

template <int NS, bool Q4>
__device__ void producer_loop(const DecodeParams& p, Shared* sh, uint8_t* ring) {
  producer_walk<NS>(p, sh, ring,
                    [](const DecodeParams& pp, const Ranges& r, const LayerW& L, int l, int s, const uint8_t*& src,
                       int& rows, int& rb) { return layer_segment<Q4>(pp, r, L, l, s, src, rows, rb); });
}

// ------------------------------------------------------------------ consumer helpers
template <int NS>
__device__ __forceinline__ const uint8_t* acquire(const DecodeParams& p, Shared* sh, uint8_t* ring, uint32_t n,
                                                  int tid, int lane) {
  const int slot = n % NS;
  if (tid == 0) trace_at(p, kTraceChunks + 4 * static_cast<int>(n) + 1);
  if (!mbar_wait(&sh->full[slot], (n / NS) & 1, &sh->abort_flag, kWaitLimitNs)) {
    if (lane == 0) {
      if (!sh->abort_flag) atomicOr(p.err, MK_DEVERR_PIPE_TIMEOUT);
      sh->abort_flag = 1;
    }
  }
  if (tid == 0) trace_at(p, kTraceChunks + 4 * static_cast<int>(n) + 2);
  return ring + static_cast<size_t>(slot) * kSlotBytes;
}
template <int NS>
__device__ __forceinline__ void release(const DecodeParams& p, Shared* sh, uint32_t& n, int lane) {
  if (threadIdx.x == 0) trace_at(p, kTraceChunks + 4 * static_cast<int>(n) + 3);
  __syncwarp();
  if (lane == 0) mbar_arrive(&sh->empty[n % NS]);
  ++n;
}

// Grid-wide barrier among the consumer threads of all CTAs (release reduction on one
// counter, acquire polling). Returns false if this CTA must stop (own or remote
// failure); the result is the same in every consumer thread.
__device__ bool grid_barrier(const DecodeParams& p, Shared* sh, unsigned k, int tid) {
  const unsigned target = k * gridDim.x;
  cons_sync(kConsumerThreads);
  if (tid == 0) {
    trace_at(p, 2 * static_cast<int>(k) - 1);
    trace_grid(p, k, 0);
    int stop = sh->abort_flag;
    if (!stop) {
      red_release_add(p.bar, 1u);
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
    }
    trace_at(p, 2 * static_cast<int>(k));
    trace_grid(p, k, 1);
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
  const float t = (lane < kConsumerWarps) ? sh->red[lane] : 0.0f;
  return warp_sum(t);
}

// Residual stream between norm phases j and j+1 (j counts every RMSNorm of the step):
// h_j = base[j % 2] + sum_c delta[j % 3][c]. The update between norms j and j+1 reduces
// its partial sums into delta[(j+1) % 3]; CTA i adds into copy i % kResCopies, so each
// address takes G / kResCopies additions instead of G (the additions of all CTAs to one
// address serialise in L2). The RMSNorm of phase j+1 adds base and the copies, and CTA 0
// writes the sum to base[(j+1) % 2]. During phase j the last kResCopies CTAs zero one
// copy each of delta[(j+2) % 3]. No CTA reads the old residual on its own critical path.
__device__ __forceinline__ float* res_base(const DecodeParams& p, int H, int j) {
  return p.hbuf + static_cast<size_t>(j % 2) * H;
}
__device__ __forceinline__ float* res_delta(const DecodeParams& p, int H, int j, int copy) {
  return p.hbuf + static_cast<size_t>(2 + (j % 3) * kResCopies + copy) * H;
}

// Norm phase j: xs = h_j / sqrt(mean(h_j^2) + eps) * gamma (fp32, kept on chip), with
// h_j = base + delta (or, for j = 0, the bf16 embedding row). All loads are issued together.
// Four consecutive weights 4g .. 4g+3 of a Q4_K-style row (144-byte super-blocks): they
// share a super-block, a sub-block and a nibble half.
__device__ __forceinline__ float4 q4_dequant4(const uint8_t* row, int g) {
  const int i = 4 * g, sb = i >> 8, w = i & 255, jb = w >> 5, t = w & 31;
  const uint8_t* blk = row + static_cast<size_t>(sb) * kQ4Block;
  const uint32_t dd = *reinterpret_cast<const uint32_t*>(blk);
  const uint64_t lo = static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 4)) |
                      (static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 8)) << 32);
  const uint64_t hi = static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 8)) |
                      (static_cast<uint64_t>(*reinterpret_cast<const uint32_t*>(blk + 12)) << 32);
  const float sc = static_cast<float>(static_cast<uint32_t>(lo >> (6 * jb)) & 63u);
  const float mm = static_cast<float>(static_cast<uint32_t>(hi >> (16 + 6 * jb)) & 63u);
  const float s = __half2float(__ushort_as_half(static_cast<unsigned short>(dd & 0xFFFFu))) * sc;
  const float mn = __half2float(__ushort_as_half(static_cast<unsigned short>(dd >> 16))) * mm;
  const uint32_t c = *reinterpret_cast<const uint32_t*>(blk + 16 + 16 * jb + (t & 15));
  const int sh = (t >= 16) ? 4 : 0;
  return make_float4(fmaf(s, static_cast<float>((c >> sh) & 15u), -mn), fmaf(s, static_cast<float>((c >> (8 + sh)) & 15u), -mn),
                     fmaf(s, static_cast<float>((c >> (16 + sh)) & 15u), -mn),
                     fmaf(s, static_cast<float>((c >> (24 + sh)) & 15u), -mn));
}

template <int MG>
__device__ __forceinline__ void rmsnorm(const DecodeParams& p, int H, int j, const uint16_t* bf_row,
                                       const uint16_t* gamma, float* xs, Shared* sh, int tid, int warp, int lane,
                                       const uint8_t* q4_row = nullptr) {
  const int ng = H / 4;
  const int cta = blockIdx.x, G = gridDim.x;
  float4 v[MG];
  if (q4_row) {
#pragma unroll
    for (int k = 0; k < MG; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) v[k] = q4_dequant4(q4_row, g);
    }
  } else if (bf_row) {
#pragma unroll
    for (int k = 0; k < MG; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) {
        const uint2 w = *reinterpret_cast<const uint2*>(bf_row + 4 * g);
        v[k] = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
      }
    }
  } else {
    const float4* hb = reinterpret_cast<const float4*>(res_base(p, H, j));
#pragma unroll
    for (int k = 0; k < MG; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) v[k] = __ldcg(hb + g);
    }
#pragma unroll
    for (int c = 0; c < kResCopies; ++c) {
      const float4* hd = reinterpret_cast<const float4*>(res_delta(p, H, j, c));
#pragma unroll
      for (int k = 0; k < MG; ++k) {
        const int g = tid + k * kConsumerThreads;
        if (g < ng) {
          const float4 d = __ldcg(hd + g);
          v[k].x += d.x; v[k].y += d.y; v[k].z += d.z; v[k].w += d.w;
        }
      }
    }
  }
  if (cta == 0) {    // materialise h_j as the next base
    float4* nb = reinterpret_cast<float4*>(res_base(p, H, j + 1));
#pragma unroll
    for (int k = 0; k < MG; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) __stcg(nb + g, v[k]);
    }
  }
  // the delta that the update after norm j+1 accumulates into: copy c is zeroed by CTA
  // G-1-c (by CTA G-1-(c mod G) on a grid smaller than kResCopies)
  for (int c = G - 1 - cta; c < kResCopies; c += G) {
    float4* z = reinterpret_cast<float4*>(res_delta(p, H, j + 2, c));
    for (int g = tid; g < ng; g += kConsumerThreads) __stcg(z + g, make_float4(0.f, 0.f, 0.f, 0.f));
    if (j == 0) {
      float4* z1 = reinterpret_cast<float4*>(res_delta(p, H, 1, c));
      for (int g = tid; g < ng; g += kConsumerThreads) __stcg(z1 + g, make_float4(0.f, 0.f, 0.f, 0.f));
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < MG; ++k) {
    const int g = tid + k * kConsumerThreads;
    if (g < ng) ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  // the sum of squares: warp sums meet in shared memory behind one named barrier, and every
  // thread adds the kConsumerWarps partials itself
  ss = warp_sum(ss);
  if (lane == 0) sh->red[warp] = ss;
  cons_sync(kConsumerThreads);
  ss = 0.f;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) ss += sh->red[w];
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + p.eps);
#pragma unroll
  for (int k = 0; k < MG; ++k) {
    const int g = tid + k * kConsumerThreads;
    if (g < ng) {
      const uint2 gw = *reinterpret_cast<const uint2*>(gamma + 4 * g);
      reinterpret_cast<float4*>(xs)[g] = make_float4(v[k].x * inv * bf16lo(gw.x), v[k].y * inv * bf16hi(gw.x),
                                                     v[k].z * inv * bf16lo(gw.y), v[k].w * inv * bf16hi(gw.y));
    }
  }
  cons_sync(kConsumerThreads);
}

// The normed input, as each lane needs it for a warp-per-row dot product: lane l holds
// x[l*8 + 256*k .. +8) for k < XK. Used (kept in registers for a whole phase) when the
// hidden size is exactly XK * 256; XK = 0 reads x from shared memory instead.
template <int XK>
struct XReg {
  float4 a[XK > 0 ? XK : 1], b[XK > 0 ? XK : 1];
};

template <int XK>
__device__ __forceinline__ void load_xreg(XReg<XK>& x, const float* xs, int H, int lane) {
#pragma unroll
  for (int k = 0; k < XK; ++k) {
    const int c = lane * 8 + 256 * k;
    x.a[k] = *reinterpret_cast<const float4*>(xs + c);
    x.b[k] = *reinterpret_cast<const float4*>(xs + c + 4);
  }
}

// Dot products of up to four bf16 rows with x, four independent accumulator chains, each
// split into even and odd positions by the packed fp32 FMA.
template <int XK>
__device__ __forceinline__ void dot4_rows(const uint8_t* p0, const uint8_t* p1, const uint8_t* p2, const uint8_t* p3,
                                          const XReg<XK>& x, const float* xs, int H, int lane, float* a) {
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  if (XK > 0) {
#pragma unroll
    for (int k = 0; k < XK; ++k) {
      const int c = lane * 8 + 256 * k;
      const uint4 w0 = *reinterpret_cast<const uint4*>(p0 + 2 * c);
      const uint4 w1 = *reinterpret_cast<const uint4*>(p1 + 2 * c);
      const uint4 w2 = *reinterpret_cast<const uint4*>(p2 + 2 * c);
      const uint4 w3 = *reinterpret_cast<const uint4*>(p3 + 2 * c);
      dot8_bf16_f2(w0, x.a[k], x.b[k], acc[0]);
      dot8_bf16_f2(w1, x.a[k], x.b[k], acc[1]);
      dot8_bf16_f2(w2, x.a[k], x.b[k], acc[2]);
      dot8_bf16_f2(w3, x.a[k], x.b[k], acc[3]);
    }
  } else {
    for (int c = lane * 8; c < H; c += 256) {
      const float4 xa = *reinterpret_cast<const float4*>(xs + c);
      const float4 xb = *reinterpret_cast<const float4*>(xs + c + 4);
      dot8_bf16_f2(*reinterpret_cast<const uint4*>(p0 + 2 * c), xa, xb, acc[0]);
      dot8_bf16_f2(*reinterpret_cast<const uint4*>(p1 + 2 * c), xa, xb, acc[1]);
      dot8_bf16_f2(*reinterpret_cast<const uint4*>(p2 + 2 * c), xa, xb, acc[2]);
      dot8_bf16_f2(*reinterpret_cast<const uint4*>(p3 + 2 * c), xa, xb, acc[3]);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) a[q] = f2_sum(acc[q]);
}

// DeltaNet conv epilogue of the in-projection: for a q/k/v row g with raw value x_t,
// store x_t into the conv history slot of this position, y = SiLU(conv) into ybuf, and
// (q and k rows) add y^2 into the CTA's per-head partial sums of squares. The taps sit
// in the 16-byte tail of the row in the chunk; the W-1 older inputs of the CTA's rows
// were staged in shared memory (chist [rows][3]).
struct ConvEpi {
  const float* chist;
  int b;            // first in-projection row of this CTA
  int W;
  int tap_off;      // byte offset of the conv taps in the row (after the weights)
  int qk_rows;      // 2 * Hd * dk
  int dk;
  int h_lo;         // first q/k head (index into [q heads | k heads]) this CTA touches
  float* ybuf;
  float* ysq;       // shared memory: y^2 of each of the CTA's rows (indexed by row - b)
};

__device__ __forceinline__ void conv_epilogue(const ConvEpi& ce, int g, float raw, const uint8_t* row, float* ringc) {
  const int lr = g - ce.b;
  const uint2 tw = *reinterpret_cast<const uint2*>(row + ce.tap_off);
  const float t0 = bf16lo(tw.x), t1 = bf16hi(tw.x), t2 = bf16lo(tw.y), t3 = bf16hi(tw.y);
  const float tcur = ce.W == 4 ? t3 : (ce.W == 3 ? t2 : t1);    // the tap of the current input
  float y = tcur * raw;
  if (ce.W > 1) y = fmaf(t0, ce.chist[lr * 3 + 0], y);
  if (ce.W > 2) y = fmaf(t1, ce.chist[lr * 3 + 1], y);
  if (ce.W > 3) y = fmaf(t2, ce.chist[lr * 3 + 2], y);
  y = siluf_(y);
  __stcg(ringc + g, raw);
  __stcg(ce.ybuf + g, y);
  ce.ysq[lr] = y * y;
}

// Warp-per-row dot products of nrows bf16 rows (stride rb bytes) with x; each warp takes
// rows warp, warp+8, warp+16, warp+24 together. Row r's value goes to lo[row_base + r]
// if row_base + r < split (through the conv epilogue when ce != nullptr), else to
// hi[row_base + r - split]; lane 0 writes it.
template <int XK>
__device__ __forceinline__ void gemv_rows(const uint8_t* chunk, int nrows, int rb, const XReg<XK>& x, const float* xs,
                                          int H, int warp, int lane, int row_base, int split, float* lo, float* hi,
                                          bool use_ce = false, ConvEpi ce = ConvEpi{}) {
  for (int r = warp; r < nrows; r += 4 * kConsumerWarps) {
    int rr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) rr[q] = (r + q * kConsumerWarps < nrows) ? r + q * kConsumerWarps : r;
    float a[4];
    dot4_rows<XK>(chunk + static_cast<size_t>(rr[0]) * rb, chunk + static_cast<size_t>(rr[1]) * rb,
                  chunk + static_cast<size_t>(rr[2]) * rb, chunk + static_cast<size_t>(rr[3]) * rb, x, xs, H, lane, a);
#pragma unroll
    for (int q = 0; q < 4; ++q) a[q] = warp_sum(a[q]);
    // lanes 0..3 finish the four rows together (one code path, one row per lane)
    const int q = lane & 3;
    const float aq = q == 0 ? a[0] : (q == 1 ? a[1] : (q == 2 ? a[2] : a[3]));
    const int rq = q == 0 ? rr[0] : (q == 1 ? rr[1] : (q == 2 ? rr[2] : rr[3]));
    if (lane < 4 && (q == 0 || rq != r)) {
      const int g = row_base + rq;
      if (g < split) {
        if (use_ce) conv_epilogue(ce, g, aq, chunk + static_cast<size_t>(rq) * rb, lo);
        else lo[g] = aq;
      } else {
        hi[g - split] = aq;
      }
    }
  }
}

// Split-K accumulate into registers: acc[out] += sum_r row_r[out] * coef[r]. Thread tid
// owns float4 groups tid, tid + 256, ... Rows are taken four at a time, loads first; each
// pair of outputs takes one packed FMA per row (the same per-element order as scalar FMAs).
template <int MG>
__device__ __forceinline__ void splitk_rows(const uint8_t* chunk, int nrows, int rb, const float* coef, int H,
                                            float4* acc, int tid) {
  const int ng = H / 4;
  if constexpr (MG >= 8) {   // the any-size instance: scalar FMAs (the packed pairs cost it registers)
    for (int r = 0; r < nrows; ++r) {
      const uint8_t* row = chunk + static_cast<size_t>(r) * rb;
      const float cf = coef[r];
#pragma unroll
      for (int k = 0; k < MG; ++k) {
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
    return;
  }
  uint64_t a2[MG][2];
#pragma unroll
  for (int k = 0; k < MG; ++k) {
    a2[k][0] = f2_pack(acc[k].x, acc[k].y);
    a2[k][1] = f2_pack(acc[k].z, acc[k].w);
  }
  int r = 0;
  for (; r + 4 <= nrows; r += 4) {
    uint2 w[4][MG];
    float cf[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      cf[q] = coef[r + q];
#pragma unroll
      for (int k = 0; k < MG; ++k) {
        const int g = tid + k * kConsumerThreads;
        if (g < ng) w[q][k] = *reinterpret_cast<const uint2*>(chunk + static_cast<size_t>(r + q) * rb + 8 * g);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint64_t c2 = f2_pack(cf[q], cf[q]);
#pragma unroll
      for (int k = 0; k < MG; ++k) {
        const int g = tid + k * kConsumerThreads;
        if (g < ng) {
          ffma2(a2[k][0], f2_pack(bf16lo(w[q][k].x), bf16hi(w[q][k].x)), c2);
          ffma2(a2[k][1], f2_pack(bf16lo(w[q][k].y), bf16hi(w[q][k].y)), c2);
        }
      }
    }
  }
  for (; r < nrows; ++r) {
    const uint8_t* row = chunk + static_cast<size_t>(r) * rb;
    const uint64_t c2 = f2_pack(coef[r], coef[r]);
#pragma unroll
    for (int k = 0; k < MG; ++k) {
      const int g = tid + k * kConsumerThreads;
      if (g < ng) {
        const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * g);
        ffma2(a2[k][0], f2_pack(bf16lo(w.x), bf16hi(w.x)), c2);
        ffma2(a2[k][1], f2_pack(bf16lo(w.y), bf16hi(w.y)), c2);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < MG; ++k) {
    const float2 lo = f2_unpack(a2[k][0]), hi = f2_unpack(a2[k][1]);
    acc[k] = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
}

// The update that follows norm j: delta[(j+1) % 3][cta % kResCopies] += this CTA's
// partial sums (fire-and-forget vector reductions).
template <int MG>
__device__ __forceinline__ void residual_add(const DecodeParams& p, int H, int j, bool has_rows, const float4* acc,
                                             int tid) {
  if (!has_rows) return;
  const int ng = H / 4;
  float4* nd = reinterpret_cast<float4*>(res_delta(p, H, j + 1, static_cast<int>(blockIdx.x) % kResCopies));
#pragma unroll
  for (int k = 0; k < MG; ++k) {
    const int g = tid + k * kConsumerThreads;
    if (g < ng) red_add_v4(nd + g, acc[k]);
  }
}

// Causal depthwise conv at channel ch over the W-slot history, then SiLU. All loads
// are issued before the arithmetic.
__device__ __forceinline__ float conv_silu_at(const DecodeParams& p, const float* ringl, const uint16_t* taps, int ch,
                                              int pos) {
  float w[kMaxConv], x[kMaxConv];
#pragma unroll
  for (int j = 0; j < kMaxConv; ++j) {
    if (j < p.convw) {
      const int src = pos - (p.convw - 1) + j;
      const int slot = ((src % p.convw) + p.convw) % p.convw;
      w[j] = bf16_to_f(taps[static_cast<size_t>(ch) * p.convw + j]);
      x[j] = __ldcg(ringl + static_cast<size_t>(slot) * p.C + ch);
    }
  }
  float y = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxConv; ++j)
    if (j < p.convw) y = fmaf(w[j], x[j], y);
  return siluf_(y);
}

// Online-softmax update of one block of np scores in sc (one warp per head).
__device__ __forceinline__ void softmax_block(float* sc, float* mlc, int grp, int np, int warp, int lane) {
  if (warp >= grp) return;
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

// ------------------------------------------------------------------ Q4_K-style rows
// One super-block (144 bytes at blk) against x. Lane l takes sub-block j = l / 4 and code
// bytes 4 (l % 4) .. +3 of it: weights 32 j + 4 (l % 4) + t (low nibbles) and
// 32 j + 16 + 4 (l % 4) + t (high nibbles), t = 0..3, whose x values are xl and xh and
// whose x sum is xsv. With w = (d sc_j) q - (dmin m_j) the lane's share of the product is
// (d sc_j) sum(q x) - (dmin m_j) sum(x); d sc_j and dmin m_j are exact in fp32.
// Lane constants of q4_part: which 32-bit words of the 6-bit field stream hold the
// lane's sc_j and m_j, and the shift inside the word pair.
struct Q4Lane {
  int j, part;
  int sc_w, sc_sh;   // sc_j at stream bit 6j
  int m_w, m_sh;     // m_j at stream bit 48 + 6j
};
__device__ __forceinline__ Q4Lane q4_lane(int lane) {
  Q4Lane q;
  q.j = lane >> 2;
  q.part = lane & 3;
  const int bs = 6 * q.j, bm = 48 + 6 * q.j;
  q.sc_w = bs >> 5;
  q.sc_sh = bs & 31;
  q.m_w = bm >> 5;
  q.m_sh = bm & 31;
  return q;
}

__device__ __forceinline__ float q4_part(const uint8_t* blk, const Q4Lane& ql, const float4& xl, const float4& xh,
                                         float xsv) {
  const uint32_t dd = *reinterpret_cast<const uint32_t*>(blk);
  const uint32_t f0 = *reinterpret_cast<const uint32_t*>(blk + 4);
  const uint32_t f1 = *reinterpret_cast<const uint32_t*>(blk + 8);
  const uint32_t f2 = *reinterpret_cast<const uint32_t*>(blk + 12);
  const uint32_t c = *reinterpret_cast<const uint32_t*>(blk + 16 + 16 * ql.j + 4 * ql.part);
  const uint32_t sc = __funnelshift_r(ql.sc_w ? f1 : f0, ql.sc_w ? f2 : f1, ql.sc_sh) & 63u;
  const uint32_t mm = __funnelshift_r(ql.m_w == 1 ? f1 : f2, ql.m_w == 1 ? f2 : 0u, ql.m_sh) & 63u;
  // small integers to float through the exponent field: 2^23 + v is exact for v < 2^23
  const float scf = __uint_as_float(0x4B000000u | sc) - 8388608.0f;
  const float mmf = __uint_as_float(0x4B000000u | mm) - 8388608.0f;
  const float s = __half2float(__ushort_as_half(static_cast<unsigned short>(dd & 0xFFFFu))) * scf;
  const float mn = __half2float(__ushort_as_half(static_cast<unsigned short>(dd >> 16))) * mmf;
  // each code q becomes the float v = 0.5 + q/256 exactly, by one byte permute of its nibble
  // under the exponent byte of 0.5 (bits 16..19 of the mantissa); the lane's 8 weights go in
  // four packed FMAs, and sum q x = 256 (sum v x) - 128 (sum x)
  const uint32_t lo = c & 0x0F0F0F0Fu, hi = (c >> 4) & 0x0F0F0F0Fu;
  constexpr uint32_t kHalfHi = 0x3F000000u;   // bytes 0..2 zero, byte 3 = 0.5's exponent byte
  uint64_t acc = 0ull;
  ffma2(acc, f2_pack(__uint_as_float(__byte_perm(lo, kHalfHi, 0x7044)), __uint_as_float(__byte_perm(lo, kHalfHi, 0x7144))),
        f2_pack(xl.x, xl.y));
  ffma2(acc, f2_pack(__uint_as_float(__byte_perm(lo, kHalfHi, 0x7244)), __uint_as_float(__byte_perm(lo, kHalfHi, 0x7344))),
        f2_pack(xl.z, xl.w));
  ffma2(acc, f2_pack(__uint_as_float(__byte_perm(hi, kHalfHi, 0x7044)), __uint_as_float(__byte_perm(hi, kHalfHi, 0x7144))),
        f2_pack(xh.x, xh.y));
  ffma2(acc, f2_pack(__uint_as_float(__byte_perm(hi, kHalfHi, 0x7244)), __uint_as_float(__byte_perm(hi, kHalfHi, 0x7344))),
        f2_pack(xh.z, xh.w));
  return fmaf(256.0f * s, f2_sum(acc), -fmaf(128.0f, s, mn) * xsv);
}

// xsum[sb * 32 + l] = the sum of the 8 x values lane l pairs with in super-block sb.
__device__ __forceinline__ void q4_xsum(const float* xs, float* xsum, int K, int tid) {
  const int n = (K >> 8) * 32;
  for (int i = tid; i < n; i += kConsumerThreads) {
    const int sb = i >> 5, l = i & 31;
    const float* xb = xs + sb * 256 + 32 * (l >> 2) + 4 * (l & 3);
    const float4 a = *reinterpret_cast<const float4*>(xb);
    const float4 b = *reinterpret_cast<const float4*>(xb + 16);
    xsum[i] = ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
  }
}

// Row products of one ring chunk of nrows Q4 rows (stride rb) with x (nsb super-blocks).
// Warp w takes super-blocks ks, ks + WK, ... (ks = w % WK) of rows rs, rs + RS, ...
// (rs = w / WK), four rows at a time; the warps' partial sums meet in qpart [WK][nrows]
// (WK * nrows <= 455 for any row length) and out(r, value) runs once per row.
template <typename Out>
__device__ __forceinline__ void gemv_rows_q4(const uint8_t* chunk, int nrows, int rb, int nsb, const float* xs,
                                             const float* xsum, float* qpart, int warp, int lane, int tid, Out&& out) {
  const int WK = nsb >= 8 ? 8 : (nsb >= 4 ? 4 : (nsb >= 2 ? 2 : 1));
  const int RS = kConsumerWarps / WK;
  const int ks = warp % WK, rs = warp / WK;
  const Q4Lane ql = q4_lane(lane);
  const int j = ql.j, part = ql.part;
  for (int r0 = rs; r0 < nrows; r0 += 4 * RS) {
    const uint8_t* rp[4];
    bool live[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + q * RS;
      live[q] = r < nrows;
      rp[q] = chunk + static_cast<size_t>(live[q] ? r : r0) * rb;
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sb = ks; sb < nsb; sb += WK) {
      const float* xb = xs + sb * 256 + 32 * j + 4 * part;
      const float4 xl = *reinterpret_cast<const float4*>(xb);
      const float4 xh = *reinterpret_cast<const float4*>(xb + 16);
      const float xsv = xsum[sb * 32 + lane];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] += q4_part(rp[q] + static_cast<size_t>(sb) * kQ4Block, ql, xl, xh, xsv);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float v = warp_sum(acc[q]);
      if (lane == 0 && live[q]) qpart[ks * nrows + r0 + q * RS] = v;
    }
  }
  cons_sync(kConsumerThreads);
  for (int r = tid; r < nrows; r += kConsumerThreads) {
    float v = 0.f;
    for (int k = 0; k < WK; ++k) v += qpart[k * nrows + r];
    out(r, v);
  }
  cons_sync(kConsumerThreads);
}

// Rows [h_b, h_e) of a Q4 projection (row stride rbk) whose K-float input sits in global
// memory (written by every CTA before the last grid barrier): stage it in xs, then the row
// products go straight into the residual delta of the update after norm j.
template <int NS>
__device__ __forceinline__ void q4_rows_to_residual(const DecodeParams& p, Shared* sh, uint8_t* ring, uint32_t& n,
                                                    const float* src, int K, int rbk, int j, float* xs, float* xsum,
                                                    float* qpart, int tid, int warp, int lane) {
  const Ranges& rg = sh->rg;
  for (int i = tid; i < K / 4; i += kConsumerThreads)
    reinterpret_cast<float4*>(xs)[i] = __ldcg(reinterpret_cast<const float4*>(src) + i);
  cons_sync(kConsumerThreads);
  q4_xsum(xs, xsum, K, tid);
  cons_sync(kConsumerThreads);
  float* dst = res_delta(p, p.H, j + 1, 0);
  const int nrows = rg.h_e - rg.h_b, rpc = kSlotBytes / rbk;
  for (int r0 = 0; r0 < nrows; r0 += rpc) {
    const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
    gemv_rows_q4(ch, min(rpc, nrows - r0), rbk, K >> 8, xs, xsum, qpart, warp, lane, tid,
                 [&](int r, float v) { __stcg(dst + rg.h_b + r0 + r, v); });
    release<NS>(p, sh, n, lane);
  }
}

// ------------------------------------------------------------------ the kernel
// HK > 0: the hidden size is exactly HK * 256 (compile-time, so the hot loops carry no
// bound checks and x lives in registers); HK = 0: any hidden size up to 8192.
template <int HK, bool Q4>
__global__ void __launch_bounds__(kThreads, 1) mk_decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int XK = HK;                                // x register groups (0: shared memory)
  constexpr int MG = HK > 0 ? (HK + 3) / 4 : 8;         // float4 groups of the hidden vector per thread
  constexpr int NS = Q4 ? 2 : kSlots;                   // ring slots (Q4 stages longer input vectors)
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  Shared* sh = reinterpret_cast<Shared*>(smem + static_cast<size_t>(NS) * kSlotBytes);
  LayerW* ltab = reinterpret_cast<LayerW*>(sh + 1);   // [n_layers] or [2] entries of p.layers
  float* xs = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ltab) +
                                       layer_table_bytes(p.ltab_full ? p.n_layers : 2));
  float* xsum = xs + p.xcap;                          // Q4: [xcap / 8] per-lane x sums
  float* qpart = xsum + (Q4 ? p.xcap / 8 : 0);        // Q4: [kQ4PartFloats] row partial sums
  float* fs = Q4 ? qpart + kQ4PartFloats : xs + p.H;  // scratch

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, G = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
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
    if (!bad) compute_ranges(p, cta, G, pos, sh->rg);
  }
  __syncthreads();
  if (sh->bad) return;

  if (warp == kConsumerWarps) {
    if (lane == 0) producer_loop<NS, Q4>(p, sh, ring);
    return;
  }

  // ---------------- consumers ----------------
  if (tid == 0) trace_at(p, 0);
  const int pos = sh->pos;
  if (p.Hkv > 0) {   // RoPE table of this position, shared by every attention layer
    for (int i = tid; i < p.D / 2; i += kConsumerThreads)
      rope_cs(static_cast<double>(pos) * p.inv_freq[i], sh->rope_c[i], sh->rope_s[i]);
  }   // published to the other consumer warps by the named barriers inside the first RMSNorm
  const Ranges& rg = sh->rg;
  const int rb = p.row_bytes;
  const int H = HK > 0 ? HK * 256 : p.H;
  const int ng = H / 4;
  uint32_t n = 0;               // next chunk index
  unsigned nbar = 0;
  constexpr int kLayerWords = static_cast<int>(sizeof(LayerW) / 4);
  if (p.ltab_full) {   // the whole table, read from layer 1 on (published by layer 0's named barriers)
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.layers);
    uint32_t* dst = reinterpret_cast<uint32_t*>(ltab);
    for (int i = tid; i < p.n_layers * kLayerWords; i += kConsumerThreads) dst[i] = __ldg(src + i);
  }

  for (int l = 0; l < p.n_layers; ++l) {
    const LayerW L = l == 0 ? p.layers[0] : ltab[p.ltab_full ? l : (l & 1)];
    // two slots: the next layer's entry is loaded now and stored into the other slot after
    // this layer's first barrier (the named barriers later in the layer publish it; that
    // slot was last read at the start of layer l - 1)
    const bool lw_mine = !p.ltab_full && l + 1 < p.n_layers && tid < kLayerWords;
    const uint32_t lw_next = lw_mine ? __ldg(reinterpret_cast<const uint32_t*>(p.layers + l + 1) + tid) : 0u;
    // ---- phase 1: pre-mixer RMSNorm + input projection (+ DeltaNet conv epilogue) ----
    if (l > 0 && !grid_barrier(p, sh, ++nbar, tid)) return;
    {
      const bool dn = (L.kind == kDeltaNet);
      const int b = dn ? rg.in_dn_b : rg.in_at_b, e = dn ? rg.in_dn_e : rg.in_at_e;
      float* ringc = p.conv_ring + static_cast<size_t>(L.idx) * p.convw * p.C + static_cast<size_t>(pos % p.convw) * p.C;
      // older conv inputs of this CTA's q/k/v rows: loads issued before the norm
      const int nconv = dn ? max(0, min(e, p.C) - b) : 0;
      const int qk_rows = 2 * p.Hd * p.dk;
      const int h_lo = (b < qk_rows) ? b / p.dk : 0;
      const int n_ss = (dn && b < qk_rows) ? (min(e, qk_rows) - 1) / p.dk - h_lo + 1 : 0;
      float th[kMaxConv - 1];
      if (tid < nconv) {
        const float* ringl = p.conv_ring + static_cast<size_t>(L.idx) * p.convw * p.C;
#pragma unroll
        for (int j = 0; j < kMaxConv - 1; ++j)
          if (j < p.convw - 1) th[j] = __ldcg(ringl + static_cast<size_t>((pos + 1 + j) % p.convw) * p.C + b + tid);
      }
      if (l == 0) {   // the residual starts as the embedding row
        if constexpr (Q4)
          rmsnorm<MG>(p, H, 0, nullptr, L.norm1, xs, sh, tid, warp, lane, p.embed + static_cast<size_t>(sh->tok) * rb);
        else
          rmsnorm<MG>(p, H, 0, reinterpret_cast<const uint16_t*>(p.embed + static_cast<size_t>(sh->tok) * rb), L.norm1,
                      xs, sh, tid, warp, lane);
      } else {
        rmsnorm<MG>(p, H, 2 * l, nullptr, L.norm1, xs, sh, tid, warp, lane);
      }
      float* ysq = fs + 3 * kConsumerThreads;
      ConvEpi ce{fs, b, p.convw, Q4 ? rb : 2 * H, qk_rows, p.dk, h_lo, p.ybuf, ysq};
      if (dn) {
        if (tid < nconv) {
#pragma unroll
          for (int j = 0; j < kMaxConv - 1; ++j)
            if (j < p.convw - 1) fs[tid * 3 + j] = th[j];
        }
        cons_sync(kConsumerThreads);
      }
      const int rb_in = dn ? rb + 16 : rb;
      const int rpc = kSlotBytes / rb_in;
      if constexpr (Q4) {
        q4_xsum(xs, xsum, H, tid);
        cons_sync(kConsumerThreads);
        for (int r0 = 0; r0 < e - b; r0 += rpc) {
          const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
          gemv_rows_q4(ch, min(rpc, e - b - r0), rb_in, H >> 8, xs, xsum, qpart, warp, lane, tid, [&](int r, float v) {
            const int g = b + r0 + r;
            if (!dn) p.z[g] = v;
            else if (g < p.C) conv_epilogue(ce, g, v, ch + static_cast<size_t>(r) * rb_in, ringc);
            else p.z[g - p.C] = v;
          });
          release<NS>(p, sh, n, lane);
        }
      } else {
        XReg<XK> xr;
        load_xreg<XK>(xr, xs, H, lane);
        for (int r0 = 0; r0 < e - b; r0 += rpc) {
          const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
          gemv_rows<XK>(ch, min(rpc, e - b - r0), rb_in, xr, xs, H, warp, lane, b + r0, dn ? p.C : kNoSplit,
                        dn ? ringc : p.z, p.z, dn, ce);
          release<NS>(p, sh, n, lane);
        }
      }
      if (n_ss > 0) {   // this CTA's share of the per-head sums of squares of q and k
        cons_sync(kConsumerThreads);
        for (int hs = warp; hs < n_ss; hs += kConsumerWarps) {
          const int hh = h_lo + hs;
          const int r_lo = max(b, hh * p.dk), r_hi = min(min(e, qk_rows), (hh + 1) * p.dk);
          float part = 0.f;
          for (int r = r_lo + lane; r < r_hi; r += 32) part += ysq[r - b];
          part = warp_sum(part);
          if (lane == 0) atomicAdd(p.ssq + (L.idx & 1) * 2 * p.Hd + hh, part);
        }
      }
    }
    if (!grid_barrier(p, sh, ++nbar, tid)) return;
    if (lw_mine) reinterpret_cast<uint32_t*>(ltab + ((l + 1) & 1))[tid] = lw_next;

    if (L.kind == kDeltaNet) {
      // ---- phase 2 (DeltaNet): conv + SiLU + L2 norm + gates, delta rule on this CTA's rows of S, out-proj split-K ----
      const int g0 = rg.dn_b, g1 = rg.dn_e, nrows = g1 - g0;
      float4 acc[MG];
#pragma unroll
      for (int k = 0; k < MG; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (nrows > 0) {
        const int h0 = g0 / p.dv, h1 = (g1 - 1) / p.dv;
        const int nh = h1 - h0 + 1;
        // scratch: qk[2 nh][dk] (q_h0, k_h0, q_h1, k_h1, ...) | ab[nh][2] | vv[nrows] | oc[nrows]
        float* qk = fs;
        float* ab = qk + nh * 2 * p.dk;
        float* vv = ab + 2 * nh;
        float* oc = vv + nrows;
        const int nqk = 2 * nh * p.dk;
        const int nitems = nqk + nrows + nh;
        const float* ssq = p.ssq + (L.idx & 1) * 2 * p.Hd;
        // One batch of loads: conv outputs of the heads' q and k, of the rows' v, the
        // gates' inputs and the per-head sums of squares; then L2-normalised q, k.
        float val[kConvItems], nrm[kConvItems];
#pragma unroll
        for (int it = 0; it < kConvItems; ++it) {
          const int i = tid + it * kConsumerThreads;
          if (i < nqk) {
            const int vec = i / p.dk, d = i % p.dk;
            const int hh = h0 + (vec >> 1);
            const int ch = ((vec & 1) ? p.Hd * p.dk : 0) + hh * p.dk + d;
            val[it] = __ldcg(p.ybuf + ch);
            nrm[it] = __ldcg(ssq + ((vec & 1) ? p.Hd : 0) + hh);
          } else if (i < nqk + nrows) {
            val[it] = __ldcg(p.ybuf + 2 * p.Hd * p.dk + g0 + (i - nqk));
          } else if (i < nitems) {
            const int hh = i - nqk - nrows;
            val[it] = __ldcg(p.z + h0 + hh);
            nrm[it] = __ldcg(p.z + p.Hd + h0 + hh);
          }
        }
#pragma unroll
        for (int it = 0; it < kConvItems; ++it) {
          const int i = tid + it * kConsumerThreads;
          if (i < nqk) {
            qk[i] = val[it] / sqrtf(nrm[it] + 1e-6f);
          } else if (i < nqk + nrows) {
            vv[i - nqk] = val[it];
          } else if (i < nitems) {
            const int hh = i - nqk - nrows;
            ab[2 * hh] = sigmoidf_(-val[it]);      // exp(-softplus(alpha))
            ab[2 * hh + 1] = sigmoidf_(nrm[it]);
          }
        }
        if (cta == G - 1) {   // the norm buffer of the next DeltaNet layer starts from zero
          float* nz = p.ssq + ((L.idx + 1) & 1) * 2 * p.Hd;
          for (int i = tid; i < 2 * p.Hd; i += kConsumerThreads) nz[i] = 0.f;
        }
        cons_sync(kConsumerThreads);
        // S rows: s = a S; u = s k; S' = s + b (v - u) k^T; o = S' q = s q + b (v - u) (k q).
        // One pass over a row gives s k, s q and k q (three interleaved warp sums), so the
        // readout needs no second reduction; each warp takes two rows at a time.
        const int srb = p.dk * 4, srpc = kSlotBytes / srb, vpl = p.dk / 32;
        for (int r0 = 0; r0 < nrows; r0 += srpc) {
          const float* ch = reinterpret_cast<const float*>(acquire<NS>(p, sh, ring, n, tid, lane));
          const int nr = min(srpc, nrows - r0);
          for (int r = warp; r < nr; r += 2 * kConsumerWarps) {
            const int rr[2] = {r, r + kConsumerWarps};
            float sv[2][8], red[2][3];
            int hl[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int rw = rr[u] < nr ? rr[u] : r;
              hl[u] = (g0 + r0 + rw) / p.dv - h0;
              const float a = ab[2 * hl[u]];
              const float* qv = qk + (2 * hl[u]) * p.dk;
              const float* kv = qk + (2 * hl[u] + 1) * p.dk;
              const float* srow = ch + static_cast<size_t>(rw) * p.dk;
              red[u][0] = red[u][1] = red[u][2] = 0.f;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                if (q < vpl) {
                  const float kk = kv[lane + 32 * q], qq = qv[lane + 32 * q];
                  sv[u][q] = a * srow[lane + 32 * q];
                  red[u][0] = fmaf(sv[u][q], kk, red[u][0]);
                  red[u][1] = fmaf(sv[u][q], qq, red[u][1]);
                  red[u][2] = fmaf(kk, qq, red[u][2]);
                }
              }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
              for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int c = 0; c < 3; ++c) red[u][c] += __shfl_xor_sync(0xFFFFFFFFu, red[u][c], o);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              if (rr[u] >= nr) continue;
              const int lr = r0 + rr[u];
              const int g = g0 + lr;
              const float coef = ab[2 * hl[u] + 1] * (vv[lr] - red[u][0]);
              const float* kv = qk + (2 * hl[u] + 1) * p.dk;
              float* sg_out = p.S + (static_cast<size_t>(L.idx) * p.Hd * p.dv + g) * p.dk;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (q < vpl) __stcg(sg_out + lane + 32 * q, fmaf(coef, kv[lane + 32 * q], sv[u][q]));
              if (lane == 0) oc[lr] = fmaf(coef, red[u][2], red[u][1]);
            }
          }
          release<NS>(p, sh, n, lane);
        }
        cons_sync(kConsumerThreads);
        if constexpr (Q4) {
          for (int lr = tid; lr < nrows; lr += kConsumerThreads) __stcg(p.obuf + g0 + lr, oc[lr]);
        } else {
          const int rpc = kSlotBytes / rb;
          for (int r0 = 0; r0 < nrows; r0 += rpc) {
            const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
            splitk_rows<MG>(ch, min(rpc, nrows - r0), rb, oc + r0, H, acc, tid);
            release<NS>(p, sh, n, lane);
          }
        }
      }
      if constexpr (Q4) {   // out-projection rows over the whole mixer output
        if (!grid_barrier(p, sh, ++nbar, tid)) return;
        q4_rows_to_residual<NS>(p, sh, ring, n, p.obuf, p.Hd * p.dv, p.rb_dn_out, 2 * l, xs, xsum, qpart, tid, warp,
                                lane);
      } else {
        residual_add<MG>(p, H, 2 * l, nrows > 0, acc, tid);
      }
    } else {
      // ---- phase 2 (attention): RoPE, KV append, split-K partial softmax over this CTA's positions ----
      if (rg.au_valid) {
        const int grp = p.Hq / p.Hkv;
        const int D = p.D, half = D / 2;
        const float scale = 1.0f / sqrtf(static_cast<float>(D));
        const int koff = p.Hq * D * (p.gated ? 2 : 1);
        const int voff = koff + p.Hkv * D;
        const int ug = rg.au_g, uj = rg.au_j, p0 = rg.au_p0, q1 = rg.au_q1;
        float* qs = fs;                       // [grp][D]  roped, pre-scaled queries
        float* sc = qs + grp * D;             // [grp][kAttnSub]
        float* mlc = sc + grp * kAttnSub;     // [grp][3]: m, l, corr
        float* kcur = mlc + 3 * grp;          // [D] current key (bf16-rounded)
        float* vcur = kcur + D;               // [D] current value (bf16-rounded)
        const bool has_cur = (rg.au_p1 == pos + 1);
        const size_t cache_g = (static_cast<size_t>(L.idx) * p.Hkv + ug) * p.max_ctx * D;
        for (int idx = tid; idx < (grp + (has_cur ? 1 : 0)) * half; idx += kConsumerThreads) {
          const int t = idx / half, i = idx % half;
          const float cs = sh->rope_c[i], sn = sh->rope_s[i];
          if (t < grp) {
            const int hq = ug * grp + t;
            const float x1 = __ldcg(p.z + hq * D + i), x2 = __ldcg(p.z + hq * D + i + half);
            qs[t * D + i] = (x1 * cs - x2 * sn) * scale;
            qs[t * D + i + half] = (x1 * sn + x2 * cs) * scale;
          } else {   // current key: rotate, then append it to the cache (bf16 here, 8-bit below)
            const float x1 = __ldcg(p.z + koff + ug * D + i), x2 = __ldcg(p.z + koff + ug * D + i + half);
            if (p.kv_q8) {   // 8-bit rows: quantised below, once the whole vector is here
              kcur[i] = x1 * cs - x2 * sn;
              kcur[i + half] = x1 * sn + x2 * cs;
            } else {
              const uint16_t k1 = f_to_bf16(x1 * cs - x2 * sn), k2 = f_to_bf16(x1 * sn + x2 * cs);
              p.kc[cache_g + static_cast<size_t>(pos) * D + i] = k1;
              p.kc[cache_g + static_cast<size_t>(pos) * D + i + half] = k2;
              kcur[i] = bf16_to_f(k1);
              kcur[i + half] = bf16_to_f(k2);
            }
          }
        }
        if (has_cur) {
          for (int d = tid; d < D; d += kConsumerThreads) {
            const float vx = __ldcg(p.z + voff + ug * D + d);
            if (p.kv_q8) {
              vcur[d] = vx;
            } else {
              const uint16_t vb = f_to_bf16(vx);
              p.vc[cache_g + static_cast<size_t>(pos) * D + d] = vb;
              vcur[d] = bf16_to_f(vb);
            }
          }
          if (p.kv_q8) {   // blocks of 32 of the key, then of the value, one warp per block
            cons_sync(kConsumerThreads);
            const int nb = D / 32;
            const size_t row = ((static_cast<size_t>(L.idx) * p.Hkv + ug) * p.max_ctx + pos) * p.kv_rb;
            for (int blk = warp; blk < 2 * nb; blk += kConsumerWarps) {
              const bool isv = blk >= nb;
              const int j = (blk - (isv ? nb : 0)) * 32 + lane;
              float* cur = isv ? vcur : kcur;
              uint8_t* dst = reinterpret_cast<uint8_t*>(isv ? p.vc : p.kc) + row;
              unsigned short sbits;
              float back;
              const int q = q8_block_lane(cur[j], sbits, back);
              dst[j] = static_cast<uint8_t>(static_cast<int8_t>(q));
              if (lane == 0) reinterpret_cast<unsigned short*>(dst + D)[j >> 5] = sbits;
              cur[j] = back;   // the current position attends to what the cache holds
            }
          }
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
        const int dpl = D / 32;
        for (int sb = p0; sb < q1; sb += kAttnSub) {
          const int np = min(kAttnSub, q1 - sb);
          {   // scores q_t . K[pp] from the K rows in shared memory, one warp per row
            const uint8_t* kb8 = acquire<NS>(p, sh, ring, n, tid, lane);
            const uint16_t* kch = reinterpret_cast<const uint16_t*>(kb8);
            for (int pp = warp; pp < np; pp += kConsumerWarps) {
              const uint16_t* krow = kch + static_cast<size_t>(pp) * D + lane * dpl;
              float kf[8];
              if (p.kv_q8) {   // lane's dpl codes lie in one block of 32: one scale
                const uint8_t* kr8 = kb8 + static_cast<size_t>(pp) * p.kv_rb;
                const float ks = __half2float(__ushort_as_half(
                    reinterpret_cast<const unsigned short*>(kr8 + D)[(lane * dpl) >> 5]));
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  kf[q] = (q < dpl) ? ks * static_cast<float>(static_cast<int8_t>(kr8[lane * dpl + q])) : 0.f;
              } else if (dpl == 8) {
                const uint4 kw = *reinterpret_cast<const uint4*>(krow);
                kf[0] = bf16lo(kw.x); kf[1] = bf16hi(kw.x); kf[2] = bf16lo(kw.y); kf[3] = bf16hi(kw.y);
                kf[4] = bf16lo(kw.z); kf[5] = bf16hi(kw.z); kf[6] = bf16lo(kw.w); kf[7] = bf16hi(kw.w);
              } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) kf[q] = (q < dpl) ? bf16_to_f(krow[q]) : 0.f;
              }
              float dd[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                dd[t] = 0.f;
                if (t < grp) {
                  const float* qv = qs + t * D + lane * dpl;
                  if (dpl == 8) {
                    const float4 qa = *reinterpret_cast<const float4*>(qv);
                    const float4 qb = *reinterpret_cast<const float4*>(qv + 4);
                    dd[t] = qa.x * kf[0] + qa.y * kf[1] + qa.z * kf[2] + qa.w * kf[3] +
                            qb.x * kf[4] + qb.y * kf[5] + qb.z * kf[6] + qb.w * kf[7];
                  } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                      if (q < dpl) dd[t] = fmaf(qv[q], kf[q], dd[t]);
                  }
                }
              }
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (t < grp) dd[t] = warp_sum(dd[t]);
              if (lane == 0) {
#pragma unroll
                for (int t = 0; t < 8; ++t)
                  if (t < grp) sc[t * kAttnSub + pp] = dd[t];
              }
            }
            release<NS>(p, sh, n, lane);
          }
          cons_sync(kConsumerThreads);
          softmax_block(sc, mlc, grp, np, warp, lane);
          cons_sync(kConsumerThreads);
          {   // values: thread d accumulates sum_pp p[pp] V[pp][d]
            const uint8_t* vb8 = acquire<NS>(p, sh, ring, n, tid, lane);
            const uint16_t* vch = reinterpret_cast<const uint16_t*>(vb8);
            if (tid < D && p.kv_q8) {   // 8-bit rows: code tid and the scale of its block
              float vsum[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) vsum[t] = 0.f;
              for (int pp = 0; pp < np; ++pp) {
                const uint8_t* vr = vb8 + static_cast<size_t>(pp) * p.kv_rb;
                const float vvv = __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(vr + D)[tid >> 5])) *
                                  static_cast<float>(static_cast<int8_t>(vr[tid]));
#pragma unroll
                for (int t = 0; t < 8; ++t)
                  if (t < grp) vsum[t] = fmaf(sc[t * kAttnSub + pp], vvv, vsum[t]);
              }
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (t < grp) oacc[t] = oacc[t] * mlc[3 * t + 2] + vsum[t];
            } else if (tid < D) {
              float vsum[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) vsum[t] = 0.f;
              int pp = 0;
              for (; pp + 4 <= np; pp += 4) {
                float v4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) v4[q] = bf16_to_f(vch[static_cast<size_t>(pp + q) * D + tid]);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                  if (t < grp) {
                    const float4 s4 = *reinterpret_cast<const float4*>(sc + t * kAttnSub + pp);
                    vsum[t] = fmaf(s4.x, v4[0], vsum[t]);
                    vsum[t] = fmaf(s4.y, v4[1], vsum[t]);
                    vsum[t] = fmaf(s4.z, v4[2], vsum[t]);
                    vsum[t] = fmaf(s4.w, v4[3], vsum[t]);
                  }
                }
              }
              for (; pp < np; ++pp) {
                const float vvv = bf16_to_f(vch[static_cast<size_t>(pp) * D + tid]);
#pragma unroll
                for (int t = 0; t < 8; ++t)
                  if (t < grp) vsum[t] = fmaf(sc[t * kAttnSub + pp], vvv, vsum[t]);
              }
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (t < grp) oacc[t] = oacc[t] * mlc[3 * t + 2] + vsum[t];
            }
            release<NS>(p, sh, n, lane);
          }
          cons_sync(kConsumerThreads);
        }
        if (has_cur) {   // the current position, from the freshly computed k, v
          if (warp < grp) {
            float d0 = 0.f;
            for (int i = lane; i < D; i += 32) d0 = fmaf(qs[warp * D + i], kcur[i], d0);
            d0 = warp_sum(d0);
            if (lane == 0) sc[warp * kAttnSub] = d0;
          }
          cons_sync(kConsumerThreads);
          softmax_block(sc, mlc, grp, 1, warp, lane);
          cons_sync(kConsumerThreads);
          if (tid < D) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              if (t < grp) oacc[t] = oacc[t] * mlc[3 * t + 2] + sc[t * kAttnSub] * vcur[tid];
          }
        }
        // partials: [hq][split][D + 2] = acc..., m, l
        if (tid < D) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (t < grp) {
              float* dst = p.part + (static_cast<size_t>(ug * grp + t) * p.max_splits + uj) * (D + 2);
              __stcg(dst + tid, oacc[t]);
            }
          }
        }
        if (tid < grp) {
          float* dst = p.part + (static_cast<size_t>(ug * grp + tid) * p.max_splits + uj) * (D + 2);
          __stcg(dst + D, mlc[3 * tid]);
          __stcg(dst + D + 1, mlc[3 * tid + 1]);
        }
      }
      if (!grid_barrier(p, sh, ++nbar, tid)) return;

      // ---- phase 3 (attention): combine partials for this CTA's columns, gate, out-proj split-K ----
      const int nsplit = rg.nsplit;
      const int c0 = rg.col_b, c1 = rg.col_e, ncol = c1 - c0;
      float4 acc[MG];
#pragma unroll
      for (int k = 0; k < MG; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ncol > 0) {
        const int hA = c0 / p.D, hB = (c1 - 1) / p.D;
        const int nhd = hB - hA + 1;
        // scratch: mv[nhd][nsplit] (m_j, then the weight e^{m_j - M} / L) | lv[nhd][nsplit] (l_j) |
        // gte[ncol] | pv[ncol][nsplit] (the splits' accumulators of this CTA's columns) | oc[ncol]
        float* mv = fs;
        float* lv = mv + nhd * nsplit;
        float* gte = lv + nhd * nsplit;
        float* pv = gte + ncol;
        float* oc = pv + ncol * nsplit;
        // everything the combine reads from the other CTAs, in one batch of loads
        const int n_ml = nhd * nsplit, n_pv = ncol * nsplit, total = 2 * n_ml + ncol + n_pv;
        for (int base = 0; base < total; base += 8 * kConsumerThreads) {
          float v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int i = base + tid + k * kConsumerThreads;
            v[k] = 0.f;
            if (i < 2 * n_ml) {
              const int i2 = i < n_ml ? i : i - n_ml;
              const int hq = hA + i2 / nsplit, j = i2 % nsplit;
              v[k] = __ldcg(p.part + (static_cast<size_t>(hq) * p.max_splits + j) * (p.D + 2) + p.D + (i < n_ml ? 0 : 1));
            } else if (i < 2 * n_ml + ncol) {
              v[k] = p.gated ? __ldcg(p.z + p.Hq * p.D + c0 + (i - 2 * n_ml)) : 0.f;
            } else if (i < total) {
              const int i3 = i - 2 * n_ml - ncol, cc = i3 / nsplit, j = i3 % nsplit;
              const int col = c0 + cc;
              v[k] = __ldcg(p.part + (static_cast<size_t>(col / p.D) * p.max_splits + j) * (p.D + 2) + col % p.D);
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int i = base + tid + k * kConsumerThreads;
            if (i < 2 * n_ml) mv[i] = v[k];   // mv and lv are contiguous
            else if (i < 2 * n_ml + ncol) gte[i - 2 * n_ml] = p.gated ? sigmoidf_(v[k]) : 1.0f;
            else if (i < total) pv[i - 2 * n_ml - ncol] = v[k];
          }
        }
        cons_sync(kConsumerThreads);
        for (int hh = warp; hh < nhd; hh += kConsumerWarps) {   // split weights e^{m_j - M} / L per head
          float M = -INFINITY;
          for (int j = lane; j < nsplit; j += 32) M = fmaxf(M, mv[hh * nsplit + j]);
          M = warp_max(M);
          float Ls = 0.f;
          for (int j = lane; j < nsplit; j += 32) Ls = fmaf(lv[hh * nsplit + j], expf(mv[hh * nsplit + j] - M), Ls);
          Ls = warp_sum(Ls);
          __syncwarp();
          for (int j = lane; j < nsplit; j += 32) mv[hh * nsplit + j] = expf(mv[hh * nsplit + j] - M) / Ls;
        }
        cons_sync(kConsumerThreads);
        for (int cc = tid; cc < ncol; cc += kConsumerThreads) {   // thread per column
          const float* wrow = mv + ((c0 + cc) / p.D - hA) * nsplit;
          const float* prow = pv + cc * nsplit;
          float o = 0.f;
          for (int j = 0; j < nsplit; ++j) o = fmaf(prow[j], wrow[j], o);
          oc[cc] = o * gte[cc];
        }
        cons_sync(kConsumerThreads);
        if constexpr (Q4) {
          for (int cc = tid; cc < ncol; cc += kConsumerThreads) __stcg(p.obuf + c0 + cc, oc[cc]);
        } else {
          const int rpc = kSlotBytes / rb;
          for (int r0 = 0; r0 < ncol; r0 += rpc) {
            const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
            splitk_rows<MG>(ch, min(rpc, ncol - r0), rb, oc + r0, H, acc, tid);
            release<NS>(p, sh, n, lane);
          }
        }
      }
      if constexpr (Q4) {
        if (!grid_barrier(p, sh, ++nbar, tid)) return;
        q4_rows_to_residual<NS>(p, sh, ring, n, p.obuf, p.Hq * p.D, p.rb_at_out, 2 * l, xs, xsum, qpart, tid, warp,
                                lane);
      } else {
        residual_add<MG>(p, H, 2 * l, ncol > 0, acc, tid);
      }
    }

    // ---- last phase: pre-MLP RMSNorm, SwiGLU gate/up, down-projection split-K ----
    if (!grid_barrier(p, sh, ++nbar, tid)) return;
    rmsnorm<MG>(p, H, 2 * l + 1, nullptr, L.norm2, xs, sh, tid, warp, lane);
    {
      const int nj = rg.f_e - rg.f_b;
      float4 acc[MG];
#pragma unroll
      for (int k = 0; k < MG; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if constexpr (Q4) {
        q4_xsum(xs, xsum, H, tid);
        cons_sync(kConsumerThreads);
      }
      if (nj > 0) {
        float* gs = fs;
        float* us = fs + nj;
        const int rpc = kSlotBytes / rb;
        if constexpr (Q4) {
          for (int half = 0; half < 2; ++half) {
            float* out = half ? us : gs;
            for (int r0 = 0; r0 < nj; r0 += rpc) {
              const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
              gemv_rows_q4(ch, min(rpc, nj - r0), rb, H >> 8, xs, xsum, qpart, warp, lane, tid,
                           [&](int r, float v) { out[r0 + r] = v; });
              release<NS>(p, sh, n, lane);
            }
          }
          for (int j = tid; j < nj; j += kConsumerThreads) __stcg(p.abuf + rg.f_b + j, siluf_(gs[j]) * us[j]);
        } else {
          XReg<XK> xr;
          load_xreg<XK>(xr, xs, H, lane);
          for (int half = 0; half < 2; ++half) {
            float* out = half ? us : gs;
            for (int r0 = 0; r0 < nj; r0 += rpc) {
              const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
              gemv_rows<XK>(ch, min(rpc, nj - r0), rb, xr, xs, H, warp, lane, r0, kNoSplit, out, out);
              release<NS>(p, sh, n, lane);
            }
          }
          cons_sync(kConsumerThreads);
          for (int j = tid; j < nj; j += kConsumerThreads) us[j] = siluf_(gs[j]) * us[j];
          cons_sync(kConsumerThreads);
          for (int r0 = 0; r0 < nj; r0 += rpc) {
            const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
            splitk_rows<MG>(ch, min(rpc, nj - r0), rb, us + r0, H, acc, tid);
            release<NS>(p, sh, n, lane);
          }
        }
      }
      if constexpr (Q4) {   // down-projection rows over the whole activation
        if (!grid_barrier(p, sh, ++nbar, tid)) return;
        q4_rows_to_residual<NS>(p, sh, ring, n, p.abuf, p.F, p.rb_ffn, 2 * l + 1, xs, xsum, qpart, tid, warp, lane);
      } else {
        residual_add<MG>(p, H, 2 * l + 1, nj > 0, acc, tid);
      }
    }
  }

  // ---------------- final norm, tied LM head, argmax ----------------
  if (!grid_barrier(p, sh, ++nbar, tid)) return;
  rmsnorm<MG>(p, H, 2 * p.n_layers, nullptr, p.norm_f, xs, sh, tid, warp, lane);
  if (cta == G - 1 && p.Hd > 0) {   // the first DeltaNet layer of the next step starts from zero norms
    for (int i = tid; i < 2 * p.Hd; i += kConsumerThreads) p.ssq[i] = 0.f;
  }
  {
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
    const int v0 = rg.v_b, nv = rg.v_e - rg.v_b;
    const int rpc = kSlotBytes / rb;
    if constexpr (Q4) {
      q4_xsum(xs, xsum, H, tid);
      cons_sync(kConsumerThreads);
      for (int r0 = 0; r0 < nv; r0 += rpc) {
        const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
        gemv_rows_q4(ch, min(rpc, nv - r0), rb, H >> 8, xs, xsum, qpart, warp, lane, tid, [&](int r, float v) {
          const int idx = v0 + r0 + r;
          if (p.logits) __stcg(p.logits + idx, v);
          if (v > bv || (v == bv && idx < bi)) {
            bv = v;
            bi = idx;
          }
        });
        release<NS>(p, sh, n, lane);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {   // warp's best (lowest index among equal values)
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
    }
    XReg<XK> xr;
    if constexpr (!Q4) load_xreg<XK>(xr, xs, H, lane);
    for (int r0 = 0; r0 < (Q4 ? 0 : nv); r0 += rpc) {
      const uint8_t* ch = acquire<NS>(p, sh, ring, n, tid, lane);
      const int nr = min(rpc, nv - r0);
      for (int r = warp; r < nr; r += 4 * kConsumerWarps) {
        int rr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) rr[q] = (r + q * kConsumerWarps < nr) ? r + q * kConsumerWarps : r;
        float a[4];
        dot4_rows<XK>(ch + static_cast<size_t>(rr[0]) * rb, ch + static_cast<size_t>(rr[1]) * rb,
                      ch + static_cast<size_t>(rr[2]) * rb, ch + static_cast<size_t>(rr[3]) * rb, xr, xs, H, lane, a);
#pragma unroll
        for (int q = 0; q < 4; ++q) a[q] = warp_sum(a[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q == 0 || rr[q] != r) {
            const int idx = v0 + r0 + rr[q];
            if (lane == 0 && p.logits) __stcg(p.logits + idx, a[q]);
            if (a[q] > bv || (a[q] == bv && idx < bi)) {
              bv = a[q];
              bi = idx;
            }
          }
        }
      }
      release<NS>(p, sh, n, lane);
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
      trace_at(p, 2 * static_cast<int>(nbar) + 1);
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

constexpr size_t kSmemLimit = 232448;

// Shared memory before the scratch: the ring, Shared, the layer table, the staged input
// vector and, with Q4 weights (2 ring slots), its per-lane sums and the row partial sums.
static size_t decode_fixed_bytes(int H, bool q4, int xcap, int ltab_entries) {
  const size_t lt = layer_table_bytes(ltab_entries);
  if (!q4) return static_cast<size_t>(kSlots) * kSlotBytes + sizeof(Shared) + lt + static_cast<size_t>(H) * 4;
  return 2 * static_cast<size_t>(kSlotBytes) + sizeof(Shared) + lt + static_cast<size_t>(xcap) * 4 +
         static_cast<size_t>(xcap / 8) * 4 + static_cast<size_t>(kQ4PartFloats) * 4;
}

size_t decode_scratch_floats(int H, bool q4, int xcap, int ltab_entries) {
  const size_t fixed = decode_fixed_bytes(H, q4, xcap, ltab_entries);
  if (fixed >= kSmemLimit) return 0;
  size_t f = (kSmemLimit - fixed) / 4;
  f &= ~static_cast<size_t>(3);
  return f > 8192 ? 8192 : f;
}

size_t decode_smem_bytes(int H, bool q4, int xcap, int ltab_entries) {
  return decode_fixed_bytes(H, q4, xcap, ltab_entries) + decode_scratch_floats(H, q4, xcap, ltab_entries) * 4;
}

int decode_max_splits(int grid, int hkv) {
  int per = grid / hkv;
  return per < 1 ? 1 : per;
}

template <int HK, bool Q4>
cudaError_t launch_hk(const DecodeParams& p, int grid, cudaStream_t s) {
  static std::atomic<uint64_t> attr_set{0};   // per device
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(mk_decode_kernel<HK, Q4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSmemLimit));
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(p.H, Q4, p.xcap, p.ltab_full ? p.n_layers : 2);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mk_decode_kernel<HK, Q4>, p);
}

cudaError_t launch_decode(const DecodeParams& p, int grid, cudaStream_t s) {
  if (p.q4) {
    if (p.H == 1024) return launch_hk<4, true>(p, grid, s);
    if (p.H == 5120) return launch_hk<20, true>(p, grid, s);
    return launch_hk<0, true>(p, grid, s);
  }
  if (p.H == 1024) return launch_hk<4, false>(p, grid, s);
  if (p.H == 256) return launch_hk<1, false>(p, grid, s);
  if (p.H == 2048) return launch_hk<8, false>(p, grid, s);
  return launch_hk<0, false>(p, grid, s);
}

}  // namespace mk
