// Internal definitions shared by the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mk {

// One-time setup per device (kernel attributes such as the dynamic shared-memory limit
// are set per device): runs setup() on the current device unless it already succeeded
// there. done holds one bit per device index below 64 (higher indices run setup every
// time). Safe to call from several threads: setup may then run twice, which is harmless
// for idempotent attribute settings.
template <typename F>
inline cudaError_t once_per_device(std::atomic<uint64_t>& done, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Persistent decode kernel geometry: 8 consumer warps do the math, one producer
// warp streams this CTA's weights through a ring of shared-memory slots with bulk
// asynchronous copies (cp.async.bulk, no multicast).
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kSlotBytes = 65536;
constexpr int kSlots = 3;
constexpr int kAttnSub = 128;         // positions per online-softmax sub-block (one 64 KB ring slot of D = 256 keys)
constexpr int kResCopies = 2;          // copies of each residual delta (CTA c adds into copy c % 2)
constexpr int kAttnMinChunk = 16;     // smallest split-K chunk of the KV cache

enum LayerKind : int { kDeltaNet = 0, kAttention = 1 };

// Per-layer device pointers into the packed weight buffer.
struct LayerW {
  int kind;
  int idx;                  // index among layers of the same kind
  const uint16_t* norm1;    // [H] bf16
  const uint16_t* norm2;    // [H] bf16
  const uint8_t* w_in;      // [in_rows][row_bytes]      (row-major [out, in]); DeltaNet rows carry a
                            // 16-byte tail with the row's conv taps (row stride row_bytes + 16)
  const uint16_t* conv;     // [C][W] bf16 (DeltaNet)
  const uint8_t* w_outT;    // [K_mix][row_bytes]       transposed: row j = column j of W_out
  const uint8_t* w_gate;    // [F][row_bytes]
  const uint8_t* w_up;      // [F][row_bytes]
  const uint8_t* w_downT;   // [F][row_bytes]           transposed: row j = column j of W_down
  // Q4_K-style weights (row-major, 144-byte super-blocks along the input dim): the
  // out-projection [H][K_mix] and the down-projection [H][F]; the fields above then hold
  // Q4 rows of the in-projection, gate and up.
  const uint8_t* w_out_q4;
  const uint8_t* w_down_q4;
};

struct DecodeParams {
  const LayerW* layers;     // device array [n_layers]
  int n_layers;
  const uint8_t* embed;     // [V][row_bytes]
  const uint16_t* norm_f;   // [H]
  const double* inv_freq;   // [D/2] RoPE frequencies theta^(-2i/D)
  // shape
  int H, V, F, Hd, dk, dv, convw, C, Hq, Hkv, D, gated, at_in_rows, max_ctx, row_bytes;
  float eps;
  // state (caller-owned)
  float* S;                 // [n_dn][Hd][dv][dk]
  float* conv_ring;         // [n_dn][W][C]
  uint16_t* kc;             // [n_at][Hkv][max_ctx] rows of kv_rb bytes: bf16 [D], or 8-bit (kv_q8)
  uint16_t* vc;
  int kv_q8;                // 1: a row is D int8 codes, then D/32 fp16 scales (blocks of 32)
  int kv_rb;                // bytes per cache row (2 * D for bf16)
  int* pos;
  int* err;
  // workspace (caller-owned)
  float* hbuf;              // [2 + 3 * kResCopies][H] residual stream: 2 bases + 3 deltas (see decode.cu)
  float* z;                 // projection outputs not kept in the conv history
  float* part;              // attention split-K partials [Hq][max_splits][D + 2]
  unsigned* bar;            // grid barrier counter
  unsigned* done;           // end-of-step arrival counter
  unsigned long long* amax; // packed (logit, index) maximum
  float* ybuf;              // [C] conv + SiLU output of the current DeltaNet layer
  float* ssq;               // [2][2*Hd] per-head sum of squares of q and k (by DeltaNet layer parity)
  int max_splits;
  // per-call io
  const int* in_token;
  int* out_token;
  float* logits;            // may be null
  // optional gate: when gate_n != null and gate_i > *gate_n the launch does nothing
  // (used to replay only the accepted prefix of a verify pass without a host round trip)
  const int* gate_n;
  int gate_i;
  // optional diagnostics: CTA 0 records %globaltimer (ns) at kernel start, at each grid
  // barrier arrival and exit, and at the end: trace[0], trace[2k-1], trace[2k], ...
  unsigned long long* trace;
  int trace_cap;
  // Q4_K-style weights: row_bytes is then (H / 256) * 144, and the out- and down-projections
  // are split over output rows (their inputs staged from obuf / abuf)
  int q4;
  int rb_dn_out, rb_at_out, rb_ffn;   // Q4 row bytes of W_out (DeltaNet, attention) and W_down
  int xcap;                           // floats of the staged input vector in shared memory
  float* obuf;                        // [max(Hd dv, Hq D)] mixer output (Q4)
  float* abuf;                        // [F] SwiGLU activation (Q4)
  int ltab_full;                      // 1: the whole layer table in shared memory, 0: two slots
};

// ltab_entries: layers whose table entries the kernel keeps in shared memory (n_layers, or 2)
size_t decode_smem_bytes(int H, bool q4, int xcap, int ltab_entries);
size_t decode_scratch_floats(int H, bool q4, int xcap, int ltab_entries);   // fp32 scratch per CTA left after the ring, the layer table, xs (and the Q4 tables)
constexpr int kQ4Block = 144;          // bytes per 256-weight super-block
constexpr int kQ4PartFloats = 512;     // shared-memory partial sums of the Q4 row products
cudaError_t launch_decode(const DecodeParams& p, int grid, cudaStream_t s);
int decode_max_splits(int grid, int hkv);

// prefill linear layers on the tensor cores (gemm.cu): C[m][n] (+)= sum_k X[m][k] W[n][k]
// with X given as its bf16 high and low parts.
constexpr int kAttnMaxSplit = 32;     // key splits per token of the prefill attention for few-token passes
constexpr int kAttnSplitRows = 148;   // tokens up to which the split workspace is sized
constexpr long long kSplitKFloats = 8ll << 20;   // split-K partial workspace of the linear layers (32 MB)

struct LinearArgs {
  const uint16_t* x_hi;     // bf16 [M][K], row stride K
  const uint16_t* x_lo;
  const void* w;            // bf16 rows of K, row stride ldw_bytes (multiple of 16)
  long long ldw_bytes;
  float* c;                 // fp32 [M][ldc]
  long long ldc;
  int M, N, K;              // K a multiple of 64
  int accumulate;
  int* err;
  float* ws = nullptr;      // optional split-K partials (when the tile grid is smaller than the GPU)
  long long ws_floats = 0;
  // SwiGLU epilogue: when set, W's rows interleave gate and up in blocks of 64 (rows 128p .. +63
  // gate features 64p .., rows 128p + 64 .. up features 64p ..), N is a multiple of 128, and
  // instead of C the kernel writes act = SiLU(gate) * up as bf16 high / low parts [M][N / 2]
  uint16_t* act_hi = nullptr;
  uint16_t* act_lo = nullptr;
};
cudaError_t launch_split_bf16(const float* x, long long ldx, uint16_t* hi, uint16_t* lo, int M, int K, cudaStream_t s);
// 2-D tensor map of a bf16 row-major [rows][cols] matrix (row stride stride_bytes), box of 64
// columns x box_rows rows, 128-byte swizzle; cached per (base, shape, box).
bool tensor_map_bf16(CUtensorMap* map, const void* base, long long rows, long long cols, long long stride_bytes,
                     int box_rows);
// flash-style causal prefill attention on the tensor cores (attn.cu)
bool attn_flash_supported(int D);
cudaError_t launch_attn_flash(const uint16_t* q_hi, const uint16_t* q_lo, const uint16_t* k, const uint16_t* vt,
                              const int* posp, int off, int T, int Hq, int Hkv, int D, int max_ctx, long long nk,
                              float* out, long long ldo, int* items, int* err, cudaStream_t s);
cudaError_t launch_linear(const LinearArgs& a, cudaStream_t s);

// repack helpers (api.cu launches them)
cudaError_t launch_transpose_bf16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t s);
cudaError_t launch_pack_rows_tail(const uint16_t* w, const uint16_t* taps, void* dst, int rows, int cols, int nconv,
                                  int W, cudaStream_t s);

}  // namespace mk
