// Host-side model handle of libmk.so (internal; the C ABI only sees an opaque pointer).
#pragma once
#include <cstdint>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

#include <string>

// Sets the thread-local message returned by mk_last_error().
void mk_set_last_error(const std::string& msg);

// Workspace of the batched prefill (rows = tokens per pass; 0 when the model has none).
struct mk_prefill_ws {
  int rows = 0;
  float* h = nullptr;        // [rows][H] residual stream
  uint16_t* xhi = nullptr;   // [rows][Kmax] bf16 high part of the current GEMM input
  uint16_t* xlo = nullptr;   // [rows][Kmax] bf16 low part
  float* z = nullptr;        // [rows][Zmax] projection outputs (at least V floats: the prompt's last logits)
  float* y = nullptr;        // [rows][Ymax] DeltaNet q k v log-a b / roped attention queries
  float* o = nullptr;        // [rows][Omax] mixer outputs
  float* u = nullptr;        // [rows][Hd dv] chunked delta rule: U
  float* w = nullptr;        // [rows][Hd dk] chunked delta rule: W
  float* p = nullptr;        // [chunks][Hd][64][64] chunked delta rule: masked decayed Q K^T
  float* gam = nullptr;      // [rows][Hd]
  float* dec = nullptr;      // [rows][Hd]
  float* apart = nullptr;    // [min(rows, kAttnSplitRows)][Hq][kAttnMaxSplit][D + 2] attention key-split partials
  float* splitk = nullptr;   // [kSplitKFloats] split-K partials of the linear layers
  unsigned long long* best = nullptr;   // [rows] packed (value, index) row maxima of the verify logits
  // flash attention on the tensor cores: V^T of one layer's kv heads [Hkv][D][nk_max]
  // (nk_max = max_ctx rounded up to 64; 0 when the head dim has no flash kernel)
  long long nk_max = 0;
  uint16_t* vt = nullptr;
  int* flash_items = nullptr;   // work counter of the persistent flash kernel (reset before each launch)
  // chunked delta rule on the tensor cores: bf16 operand images [chunks][Hd][bytes per image]
  uint8_t* img = nullptr;
  // 8-bit KV cache: one attention layer's K and V read back as bf16 [2][Hkv][max_ctx][D]
  uint16_t* kvd = nullptr;
};

struct mk_prefill_layer {   // K-major copies of the projections the decode kernel keeps transposed
  const uint8_t* w_out;      // [H][K_mix] bf16
  const uint8_t* w_down;     // [H][F] bf16
  const uint8_t* w_gu;       // [2F][H] bf16: gate and up rows interleaved in blocks of 64 (SwiGLU epilogue)
};

// What a verify pass keeps so that the recurrent state can be committed to any accepted
// prefix afterwards (per DeltaNet layer, per token of the pass).
// Sampled verify scratch (double stats of mk_verify_ws): per-slice row statistics, the
// decision, and the chunk sums of the stopping row.
constexpr int kSampSlices = 24;      // CTAs per logits row for the row statistics
constexpr int kDrawChunks = 4096;    // slices of the stopping row for the draw
constexpr int kDrawGroup = 64;       // chunks per group of the draw's walk
struct SampDecision {
  double M;                          // maximum of the stopping row
  int n;                             // drafts kept
  int excl;                          // the rejected draft (-1: none)
};
inline size_t samp_scratch_bytes(int rows) {
  return static_cast<size_t>(rows) * kSampSlices * 2 * sizeof(double) + sizeof(SampDecision) +
         static_cast<size_t>(kDrawChunks) * sizeof(double);
}

struct mk_verify_ws {
  int rows = 0;              // tokens per pass it holds (max_draft + 1); 0: no batched verify
  float* delta = nullptr;    // [n_dn][rows][Hd dv] delta-rule updates
  float* k = nullptr;        // [n_dn][rows][Hd dk] normalised keys
  float* g = nullptr;        // [n_dn][rows][Hd] cumulative log decay inside the pass
  float* raw = nullptr;      // [n_dn][rows][C] conv inputs
  float* logits = nullptr;   // [rows][V]
  int32_t* greedy = nullptr; // [rows]
  double* stats = nullptr;   // samp_scratch_bytes(rows): sampled verify scratch
};

// Batched prefill of n tokens at the device position: every layer, no logits.
int mk_prefill_batched(mk_model* m, const int32_t* d_tokens, int n, cudaStream_t s);
int mk_prefill_tail(mk_model* m, int n, float* d_logits, int32_t* d_next_token, cudaStream_t s);
// Verify pass of K+1 tokens in one pass over the weights, acceptance, and commit of the
// accepted prefix (DeltaNet state and conv history rebuilt from the saved updates).
// Greedy acceptance when d_uniforms is NULL, else sampled acceptance at `temperature`
// with the 2(K+1) uniforms of d_uniforms.
int mk_verify_batched(mk_model* m, const int32_t* d_tokens, int K, int32_t* d_n_accepted, int32_t* d_out_tokens,
                      float* d_logits, cudaStream_t s, float temperature = 1.0f, const float* d_uniforms = nullptr);

// A captured verify pass (CUDA graph) and the arguments it was captured with: passes with
// the same arguments replay it on the model's own stream, ordered after and before the
// caller's stream by two events.
struct mk_verify_graph {
  cudaGraphExec_t exec = nullptr;
  cudaStream_t stream = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  const int32_t* tokens = nullptr;
  int K = -1;
  int32_t* n_accepted = nullptr;
  int32_t* out_tokens = nullptr;
  float* logits = nullptr;
  float temperature = 0.f;
  const float* uniforms = nullptr;
  int seen = 0;            // uncaptured passes run with these arguments
  int64_t launches = 0;    // kernel launches in one pass
};

struct mk_model {
  mk_config cfg;
  mk_sizes sz;
  uint8_t* packed;
  uint8_t* state;
  uint8_t* ws;
  int grid;
  int device;
  mk::DecodeParams base;
  std::vector<mk::LayerW> layers_host;
  int64_t launches;
  int64_t pos_hint;      // host shadow of the device position (calls through this handle); a lower bound
  int64_t pos_max;       // an upper bound of the device position (verify passes commit 1..K+1 tokens)
  // workspace sub-buffers used by the host-side drivers
  int32_t* ws_tok;       // [max_ctx + 8] token staging for prefill / generate
  int32_t* ws_g;         // [max_draft + 1] greedy tokens of a verify pass
  int32_t* ws_n;         // accepted-draft count of the last verify pass
  uint8_t* ws_snap;      // DeltaNet S + conv history + pos snapshot for verify
  size_t snap_S_bytes, snap_conv_bytes;
  size_t step_scratch_bytes;   // leading part of the workspace one decode step uses
  mk_prefill_ws pf;
  std::vector<mk_prefill_layer> pf_layers;
  mk_verify_ws vf;
  mk_verify_graph vgraph;
  ~mk_model() {
    if (vgraph.exec) cudaGraphExecDestroy(vgraph.exec);
    if (vgraph.ev_in) cudaEventDestroy(vgraph.ev_in);
    if (vgraph.ev_out) cudaEventDestroy(vgraph.ev_out);
    if (vgraph.stream) cudaStreamDestroy(vgraph.stream);
  }
};
