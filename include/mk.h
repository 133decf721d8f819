/*
 * mk.h -- C ABI of the hybrid Gated-DeltaNet + attention megakernel library (libmk.so).
 *
 * What it computes: batch-1 autoregressive inference of a hybrid language model
 * whose layers are either Gated DeltaNet mixers (linear attention whose state
 * evolves by a learned recurrence) or full softmax attention, each followed by a
 * SwiGLU MLP, as in the Hacker News post on the fused 24-layer Qwen3.5-0.8B
 * megakernel (design bullets: a single launch per forward pass, bf16 storage with
 * fp32 sums, cooperative grid syncs in place of kernel boundaries) and
 * in the open-jet Qwen3.8-27B megakernel follow-up (speculative verify of several
 * drafted tokens per pass, exact greedy acceptance or sampling that keeps the model's
 * distribution, type-checked tensor loading).
 *
 * Per token (pre-norm residual blocks, no biases; weights bf16 or 4-bit blocks, every
 * activation fp32 -- the batched passes' tensor-core products take each fp32 input as a
 * bf16 high + low pair, about 16 mantissa bits -- and the KV cache entries stored in bf16):
 *   h = E[tok]
 *   per layer:  x = RMSNorm(h) * g1
 *     DeltaNet: [q;k;v;alpha;beta] = W_in x; q,k,v = SiLU(causal depthwise conv_W);
 *               q,k L2-normalised per head; a = exp(-softplus(alpha)); b = sigmoid(beta);
 *               S = a S (I - b k k^T) + b v k^T;  o = S q;     h += W_out o
 *     attention:[q;gate;k;v] = W_in x; RoPE(q,k) (half split, theta); append bf16 k,v;
 *               o = softmax(q K^T / sqrt(D)) V per query head (GQA);
 *               o *= sigmoid(gate) (if gated);                  h += W_out o
 *     MLP:      x = RMSNorm(h) * g2;  h += W_down (SiLU(W_gate x) * (W_up x))
 *   logits = E (RMSNorm(h) * g_f)  (tied embedding);  next = argmax, lowest index on ties
 *
 * Memory ownership: the caller allocates ALL device memory (packed weights, state,
 * workspace) and passes raw device pointers; the library never allocates device
 * memory and never synchronises a stream except in mk_sync_status and mk_generate.
 * A model handle borrows the three buffers until mk_free.
 *
 * Streams: every compute call is asynchronous on the given cudaStream_t (passed as
 * void*; NULL = the legacy default stream). Token ids stay on the device between
 * calls: mk_decode_step reads its input token from device memory.
 *
 * Errors: every int-returning call returns MK_OK (0) or a negative MK_ERR_* code;
 * mk_last_error() then returns a thread-local message. Errors detected on the
 * device (a barrier or pipeline wait that gave up) are latched in the device error
 * word of the state buffer; mk_sync_status() reads it, and every later compute call
 * returns MK_ERR_DEVICE until mk_reset_state() clears it.
 */
#ifndef MK_H_
#define MK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---- */
#define MK_OK               0
#define MK_ERR_ARG         -1   /* null pointer, bad count, bad draft length, unsupported shape */
#define MK_ERR_TENSOR      -2   /* missing / unknown / duplicate tensor name, wrong dtype, shape, size or alignment */
#define MK_ERR_CAPACITY    -3   /* position + tokens would exceed max_ctx */
#define MK_ERR_CUDA        -4   /* a CUDA runtime call failed (message holds cudaGetErrorString) */
#define MK_ERR_DEVICE      -5   /* the device error word is set (a bounded wait gave up); reset needed */
#define MK_ERR_RESIDENCY   -6   /* the persistent grid cannot be co-resident on this device */

/* ---- device error word bits (state buffer, int32 at offset off_err) ---- */
#define MK_DEVERR_BARRIER_TIMEOUT   0x1   /* a grid barrier wait exceeded its time limit */
#define MK_DEVERR_PIPE_TIMEOUT      0x2   /* a shared-memory pipeline wait exceeded its limit */
#define MK_DEVERR_BAD_TOKEN         0x4   /* an input token id was outside [0, vocab) */
#define MK_DEVERR_CAPACITY          0x8   /* the device-side position reached max_ctx */

/* ---- tensor dtypes ---- */
#define MK_DT_BF16  1     /* 2 bytes per element, bf16 bit patterns */
#define MK_DT_F32   2
#define MK_DT_Q4K   3     /* 144-byte super-blocks of 256 weights along the last dim (see below) */

/* ---- weight formats ---- */
#define MK_W_BF16   0     /* every tensor bf16 */
#define MK_W_Q4K    1     /* 2-D projections (incl. the tied embedding) as MK_DT_Q4K; conv taps, gains bf16 */

/* ---- KV-cache entry formats ---- */
#define MK_KV_BF16  0     /* one bf16 per entry */
#define MK_KV_Q8    1     /* per (layer, kv head, position) row: D int8 codes, then D/32 fp16 scales,
                             the row padded to a multiple of 16 bytes; entry j reads back as
                             scale[j / 32] * code[j]; blocks of 32 with scale = max|x| / 127 and
                             code = round(x / scale) (float32, ties to even); the 8-bit cache the
                             open-jet follow-up's limits section uses for long contexts */

#define MK_MAX_LAYERS 128

/* Model shape. Plain data; copied at load. */
typedef struct mk_config {
  int32_t n_layers;
  char    pattern[MK_MAX_LAYERS + 1]; /* 'D' (Gated DeltaNet) or 'A' (attention) per layer, NUL-terminated */
  int32_t hidden;          /* H, multiple of 256, <= 8192 */
  int32_t vocab;           /* V */
  float   rms_eps;         /* RMSNorm epsilon */
  int32_t dn_heads;        /* DeltaNet heads Hd */
  int32_t dn_dk;           /* key dim per head (multiple of 32, <= 256) */
  int32_t dn_dv;           /* value dim per head (<= 256) */
  int32_t conv_width;      /* causal depthwise conv width W (2..4) */
  int32_t at_q_heads;      /* attention query heads Hq */
  int32_t at_kv_heads;     /* attention key/value heads Hkv (Hq % Hkv == 0) */
  int32_t at_head_dim;     /* D (multiple of 64, <= 256) */
  float   rope_theta;      /* RoPE base */
  int32_t at_out_gate;     /* 1: o *= sigmoid(gate rows of W_in) */
  int32_t ffn;             /* MLP intermediate size F */
  int32_t weight_format;   /* MK_W_BF16 or MK_W_Q4K */
  int32_t max_ctx;         /* KV-cache capacity in positions */
  int32_t max_draft;       /* largest K accepted by mk_verify_drafts */
  int32_t kv_format;       /* MK_KV_BF16 or MK_KV_Q8 */
} mk_config;

/* One input weight tensor (device memory, caller-owned, read during mk_load_weights only).
 * Names and shapes (row-major, [out, in] for projections):
 *   "embed"                 [V, H]            tied input embedding and LM head
 *   "norm_f"                [H]               final RMSNorm gain
 *   "layers.{l}.norm1"      [H]               pre-mixer RMSNorm gain
 *   "layers.{l}.norm2"      [H]               pre-MLP RMSNorm gain
 *   DeltaNet layer l:
 *   "layers.{l}.dn.w_in"    [Hd*(2dk+dv) + 2Hd, H]  rows q | k | v | alpha | beta
 *   "layers.{l}.dn.conv"    [Hd*(2dk+dv), W]  conv taps; column W-1 multiplies the current token
 *   "layers.{l}.dn.w_out"   [H, Hd*dv]
 *   attention layer l:
 *   "layers.{l}.attn.w_in"  [Hq*D*(1+gate) + 2*Hkv*D, H]  rows q | gate (if any) | k | v
 *   "layers.{l}.attn.w_out" [H, Hq*D]
 *   every layer:
 *   "layers.{l}.mlp.w_gate" [F, H]   "layers.{l}.mlp.w_up" [F, H]   "layers.{l}.mlp.w_down" [H, F]
 * dtype MK_DT_BF16, or MK_DT_Q4K for 2-D projections under MK_W_Q4K (then `bytes` =
 * rows * cols/256 * 144). `data` must be 16-byte aligned.
 *
 * Q4_K-style super-block (144 bytes for 256 consecutive weights of a row):
 *   [0:2] d (fp16)  [2:4] dmin (fp16)  [4:16] sixteen 6-bit fields, little-endian bit
 *   stream: sc_0..sc_7, m_0..m_7  [16:144] codes; sub-block j uses bytes 16+16j..16+16j+15,
 *   byte t holds weight 32j+t (low nibble) and 32j+t+16 (high nibble).
 *   w = (d * sc_j) * q - (dmin * m_j).
 */
typedef struct mk_tensor {
  const char* name;
  int32_t     dtype;
  int32_t     ndim;
  int64_t     shape[4];
  const void* data;        /* device pointer */
  uint64_t    bytes;
} mk_tensor;

/* Sizes of the caller-owned device buffers, and the layout of the state buffer so
 * callers can snapshot, restore or seed it with plain device copies.
 * State buffer (all offsets in bytes, 256-byte aligned):
 *   off_S    fp32 [n_dn][Hd][dv][dk]     DeltaNet states S (row i of head h = value dim i)
 *   off_conv fp32 [n_dn][W][Hd*(2dk+dv)] raw conv inputs; slot (p mod W) holds position p
 *   off_k    [n_at][Hkv][max_ctx] rows of the key cache (RoPE applied): bf16 [D], or with
 *            MK_KV_Q8 the 8-bit row format above (kv_row_bytes in mk_sizes)
 *   off_v    the value cache, same layout
 *   off_pos  int32   number of positions consumed so far
 *   off_err  int32   device error word (MK_DEVERR_* bits)
 */
typedef struct mk_sizes {
  uint64_t packed_bytes;
  uint64_t state_bytes;
  uint64_t workspace_bytes;
  uint64_t off_S, off_conv, off_k, off_v, off_pos, off_err;
  int32_t  grid_ctas;      /* persistent CTAs the decode kernel will use on the current device */
  int32_t  kv_row_bytes;   /* bytes per (layer, kv head, position) row of the KV cache */
  int32_t  layer_table_entries;  /* layer-table entries the decode kernel keeps in shared memory:
                                    n_layers when the whole table fits beside its scratch, else 2
                                    (each layer's entry is then fetched during the layer before) */
} mk_sizes;

typedef struct mk_model mk_model;   /* opaque host-side handle */

/* Validate cfg and report buffer sizes for the current CUDA device. */
int mk_query_sizes(const mk_config* cfg, mk_sizes* out);

/* Check every tensor (name, dtype, shape, byte size, alignment; none missing, none
 * unknown, none twice; the open-jet follow-up reports that its loader type-checks every
 * tensor), then repack them into d_packed (asynchronously on `stream`), zero the state and the
 * workspace, and return a handle in *out. The input tensors may be freed once the
 * stream has passed this call. */
int mk_load_weights(const mk_config* cfg, const mk_tensor* tensors, int32_t n_tensors,
                    void* d_packed, void* d_state, void* d_workspace, void* stream,
                    mk_model** out);

/* Zero S, conv history, KV cache, position and device error word. */
int mk_reset_state(mk_model* m, void* stream);

/* Consume n prompt tokens (device int32[n]) at positions pos..pos+n-1.
 * d_last_logits: device float[V] or NULL -- logits after the last token.
 * d_next_token:  device int32 or NULL -- greedy token after the last prompt token. */
int mk_prefill(mk_model* m, const int32_t* d_tokens, int32_t n,
               float* d_last_logits, int32_t* d_next_token, void* stream);

/* Set the device position (number of positions already in the state), e.g. after
 * seeding S, conv history and KV cache directly. 0 <= pos <= max_ctx. */
int mk_set_position(mk_model* m, int32_t pos, void* stream);

/* One decode step, one kernel launch: read the token at d_in_token (device), run all
 * layers at position pos, write the greedy next token to d_out_token (device; may
 * equal d_in_token) and, if d_logits != NULL, the fp32 logits [V]; pos += 1. */
int mk_decode_step(mk_model* m, const int32_t* d_in_token, int32_t* d_out_token,
                   float* d_logits, void* stream);

/* The same decode step as mk_decode_step, but its scratch memory (the barrier words,
 * residual stream, projection outputs and attention partials that the step uses
 * internally) lives in a fixed 4 MiB device array inside this library instead of the
 * workspace given to mk_load_weights. It is for callers that cannot allocate device
 * memory at the point where they step the model: hard real-time loops that must not
 * stall on cudaMalloc's implicit synchronisation, or hosts that keep a fixed
 * device-memory budget. It calls no cudaMalloc, cudaFree or other allocating routine.
 * Call it from ordinary host code, like every other entry point: not from a CUDA host
 * callback or stream-ordered host function, where CUDA allows no CUDA call at all.
 * The paper has no counterpart to it.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current. CUDA loads a library's device code lazily by default, so
 *   that first call also loads and reserves the array on the device; make it outside any
 *   latency-critical region and before any stream capture. The array then stays reserved
 *   until the process exits.
 * - The scratch a step needs does not depend on the context length: about 0.7 MB for the
 *   0.8B-shaped model, 1.3 MB for the 27B-shaped one.
 * - Every call shares the array and it keeps the last call's contents: each call clears,
 *   on `stream`, the part that must start at zero. Calls whose kernels overlap on the
 *   GPU (other streams, other threads, other models) race on the array.
 * - Returns MK_ERR_CAPACITY if the model's per-step scratch exceeds 4 MiB or the context
 *   is full; MK_ERR_ARG if the current device is not the model's; otherwise the same
 *   arguments, results and errors as mk_decode_step. */
int mk_decode_step_noalloc(mk_model* m, const int32_t* d_in_token, int32_t* d_out_token,
                           float* d_logits, void* stream);

/* Speculative verify (exact greedy acceptance, the open-jet follow-up's speed section):
 * d_tokens = [last committed token, d_1 .. d_K] (device int32[K+1]), 1 <= K <= max_draft.
 * Scores all K+1 positions; n = the longest prefix with d_j equal to the greedy token
 * after position j-1; commits d_1..d_n and the bonus greedy token g_n, leaving the
 * state exactly as if [last, d_1..d_n] had been decoded one by one.
 * Writes *d_n_accepted = n (device int32), d_out_tokens[0..n] = d_1..d_n, g_n
 * (device int32[K+1]; entries past n are left as is) and, if non-NULL, d_logits
 * [(K+1) x V] fp32 for every scored position.
 * With the batched verify workspace (max_draft + 1 <= 64 and a prefill workspace) the pass
 * runs as ~10 kernels per layer; the drafts are first copied into the model's own buffer,
 * and from the second pass with the same K, d_n_accepted, d_out_tokens, d_logits (and, in
 * sampling mode, temperature and d_uniforms) the pass is replayed as one CUDA graph on a
 * stream the model owns, ordered after and before `stream` by two events (the graph, the
 * stream and the events are released by mk_free; models with the 8-bit KV cache always
 * launch kernel by kernel). The first such call must not be made while `stream` is being
 * captured. */
int mk_verify_drafts(mk_model* m, const int32_t* d_tokens, int32_t K, int32_t* d_n_accepted,
                     int32_t* d_out_tokens, float* d_logits, void* stream);

/* Speculative verify in sampling mode (the open-jet follow-up's speed section: with
 * sampling, speculation keeps the distribution the model has without drafts). Standard
 * speculative sampling with each draft a point mass: with p_i = softmax(z_i / temperature)
 * the model's distribution after input i of [last, d_1 .. d_K],
 *   - d_{i+1} is kept iff d_uniforms[2i] < p_i(d_{i+1}), for i = 0, 1, ... until the first
 *     rejection or until all K are kept (n = the number kept);
 *   - the token after them is drawn from p_n with d_{n+1} removed and the rest
 *     renormalised (n < K), or from p_K (n = K): the smallest token index whose running
 *     weight exceeds d_uniforms[2n + 1] times the total.
 * d_uniforms: device float[2(K+1)], each in [0, 1), caller-drawn (the library draws no
 * random numbers); other values give a valid token id but no distribution guarantee.
 * temperature: > 0 and finite (MK_ERR_ARG otherwise). The weights, sums and comparisons
 * are float64, from the float32 logits.
 * Outputs, commit of the accepted prefix and the state afterwards as mk_verify_drafts.
 * Needs the batched verify workspace (max_draft + 1 <= 64 and a prefill workspace),
 * MK_ERR_CAPACITY otherwise. */
int mk_verify_drafts_sampled(mk_model* m, const int32_t* d_tokens, int32_t K, float temperature,
                             const float* d_uniforms, int32_t* d_n_accepted, int32_t* d_out_tokens,
                             float* d_logits, void* stream);

/* Convenience end-to-end call with HOST buffers: copy h_prompt[n_prompt] to the
 * device, prefill it, greedily generate n_new tokens, copy them to h_out[n_new].
 * Synchronises `stream` before returning. Uses the workspace; no allocation. */
int mk_generate(mk_model* m, const int32_t* h_prompt, int32_t n_prompt,
                int32_t* h_out, int32_t n_new, void* stream);

/* Synchronise `stream`, then return MK_OK, MK_ERR_DEVICE (device error word set; the
 * word itself is stored to *dev_err if non-NULL) or MK_ERR_CUDA. */
int mk_sync_status(mk_model* m, void* stream, int32_t* dev_err);

/* Diagnostics: while d_trace (device uint64[capacity]) is non-NULL, every decode launch
 * has CTA 0 record its SM cycle counter at its start (entry 0), at the arrival at and
 * exit from grid barrier k (entries 2k-1, 2k) and when its LM-head slice is done
 * (entry 2*n_barriers+1); from entry 512 on, chunk n of its weight stream was issued
 * (512+4n), consumer warp 0 started waiting for it (513+4n), had it (514+4n) and was
 * done with it (515+4n; chunks past entry 16383 are not recorded); from entry 16384 on,
 * every CTA c records the global timer (ns) when it arrives at grid barrier k
 * (16384 + 2(k*grid + c)) and when it leaves it (the entry after). Entries at or past `capacity` are not written. Pass NULL to stop. The
 * buffer stays the caller's. */
int mk_phase_trace(mk_model* m, uint64_t* d_trace, int32_t capacity);

/* Number of kernel launches issued by this handle so far (decode, prefill, verify,
 * repack); used to report launch counts. */
int64_t mk_launch_count(const mk_model* m);

/* Tensor-core linear layer, the building block of the prefill's projections (also
 * usable on its own): for m < M, n < N
 *     C[m][n] = sum_k X[m][k] * W[n][k]         (accumulate == 0)
 *     C[m][n] += sum_k X[m][k] * W[n][k]        (accumulate != 0)
 * d_x      device fp32, row-major [M][ldx] (ldx >= K). Split on the device into bf16
 *          high and low parts (X = hi + lo to about 16 bits of X's mantissa), each
 *          multiplied by W on the tensor cores into one fp32 accumulator.
 * d_w      device bf16, N rows of K weights, row stride ldw_bytes (a multiple of 16,
 *          >= 2K); 16-byte aligned.
 * d_c      device fp32, row-major [M][ldc] (ldc >= N).
 * K        a positive multiple of 64; M, N >= 0 (0 does nothing).
 * d_scratch, scratch_bytes: device buffer of at least 4*M*K bytes, 16-byte aligned,
 *          used for the bf16 parts of X; the caller owns it.
 * d_err    device int32 error word; a timed-out wait ORs MK_DEVERR_PIPE_TIMEOUT into it.
 * Asynchronous on `stream`. Returns MK_OK, MK_ERR_ARG (sizes, NULL or misaligned
 * pointers; nothing is launched) or MK_ERR_CUDA. */
int mk_linear(const float* d_x, int64_t ldx, int32_t M, int32_t K, const void* d_w, int64_t ldw_bytes, int32_t N,
              float* d_c, int64_t ldc, int32_t accumulate, void* d_scratch, size_t scratch_bytes, int32_t* d_err,
              void* stream);

/* Thread-local description of the last nonzero return on this thread. */
const char* mk_last_error(void);

/* Release the host-side handle (device buffers stay the caller's). */
void mk_free(mk_model* m);

#ifdef __cplusplus
}
#endif
#endif /* MK_H_ */
