// C ABI of libmk.so: validation, weight repacking, state/workspace layout and launches.
// Every step of the forward pass runs in this library's kernels; the caller only
// provides device memory and a stream.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

}  // namespace

void mk_set_last_error(const std::string& msg) { g_err = msg; }

namespace {

int cuda_fail(cudaError_t e, const char* what) {
  g_err = std::string(what) + ": " + cudaGetErrorString(e);
  return MK_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

constexpr size_t kResetBytes = 4096;   // workspace head: barrier/arrival/argmax words, per-head sums of squares

struct Expect {
  int dtype;
  int ndim;
  int64_t shape[2];
  uint64_t bytes;
};

int n_kind(const mk_config& c, char k) {
  int n = 0;
  for (int i = 0; i < c.n_layers; ++i) n += (c.pattern[i] == k);
  return n;
}

}  // namespace

#include "mk_model.h"

namespace mk {

__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int rows,
                                      int cols) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[static_cast<size_t>(r) * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[static_cast<size_t>(c) * rows + r] = tile[threadIdx.x][i];
  }
}

// Row r of dst = row r of w (cols bf16) followed by a 16-byte tail: the W conv taps of
// channel r (bf16) when r < nconv, zeros otherwise.
__global__ void pack_rows_tail_kernel(const uint16_t* __restrict__ w, const uint16_t* __restrict__ taps,
                                      uint16_t* __restrict__ dst, int rows, int cols, int nconv, int W) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  const int stride = cols + 8;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) dst[static_cast<size_t>(r) * stride + c] = w[static_cast<size_t>(r) * cols + c];
  if (threadIdx.x < 8) {
    const int j = threadIdx.x;
    dst[static_cast<size_t>(r) * stride + cols + j] = (r < nconv && j < W) ? taps[static_cast<size_t>(r) * W + j] : 0;
  }
}

// Q4 rows: row r of dst = the rbytes bytes of row r of w followed by the 16-byte taps tail.
__global__ void pack_q4_rows_tail_kernel(const uint32_t* __restrict__ w, const uint16_t* __restrict__ taps,
                                         uint32_t* __restrict__ dst, int rows, int rwords, int nconv, int W) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  const int stride = rwords + 4;
  for (int c = threadIdx.x; c < rwords; c += blockDim.x) dst[static_cast<size_t>(r) * stride + c] = w[static_cast<size_t>(r) * rwords + c];
  if (threadIdx.x < 8) {
    const int j = threadIdx.x;
    uint16_t* tail = reinterpret_cast<uint16_t*>(dst + static_cast<size_t>(r) * stride + rwords);
    tail[j] = (r < nconv && j < W) ? taps[static_cast<size_t>(r) * W + j] : 0;
  }
}

cudaError_t launch_pack_q4_rows_tail(const void* w, const uint16_t* taps, void* dst, int rows, int rbytes, int nconv,
                                     int W, cudaStream_t s) {
  pack_q4_rows_tail_kernel<<<rows, 256, 0, s>>>(static_cast<const uint32_t*>(w), taps, static_cast<uint32_t*>(dst), rows,
                                                rbytes / 4, nconv, W);
  return cudaGetLastError();
}

cudaError_t launch_pack_rows_tail(const uint16_t* w, const uint16_t* taps, void* dst, int rows, int cols, int nconv,
                                  int W, cudaStream_t s) {
  pack_rows_tail_kernel<<<rows, 256, 0, s>>>(w, taps, static_cast<uint16_t*>(dst), rows, cols, nconv, W);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  transpose_bf16_kernel<<<grid, block, 0, s>>>(src, dst, rows, cols);
  return cudaGetLastError();
}

__global__ void set_int_kernel(int* p, int v) { *p = v; }

// Longest-prefix greedy acceptance of one verify pass.
// tokens = [last, d_1..d_K], g[i] = greedy token after input i (i = 0..K).
__global__ void accept_kernel(const int* tokens, const int* g, int K, int* n_out, int* n_acc, int* out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int n = 0;
  while (n < K && tokens[1 + n] == g[n]) ++n;
  for (int i = 0; i < n; ++i) out[i] = tokens[1 + i];
  out[n] = g[n];
  *n_out = n;
  *n_acc = n;
}

}  // namespace mk

namespace {

// Bytes per (layer, kv head, position) row of the KV cache.
size_t kv_row_bytes(const mk_config& c) {
  const size_t D = static_cast<size_t>(c.at_head_dim);
  if (c.kv_format == MK_KV_Q8) return (D + D / 16 + 15) / 16 * 16;   // codes, fp16 scales, padding
  return 2 * D;
}

int check_config(const mk_config* c) {
  if (!c) return fail(MK_ERR_ARG, "config is NULL");
  if (c->n_layers < 1 || c->n_layers > MK_MAX_LAYERS) return fail(MK_ERR_ARG, "n_layers out of range");
  if (static_cast<int>(strnlen(c->pattern, MK_MAX_LAYERS + 1)) != c->n_layers)
    return fail(MK_ERR_ARG, "pattern length differs from n_layers");
  for (int i = 0; i < c->n_layers; ++i)
    if (c->pattern[i] != 'D' && c->pattern[i] != 'A') return fail(MK_ERR_ARG, "pattern must hold only 'D' and 'A'");
  if (c->hidden <= 0 || c->hidden % 8 || c->hidden > 8192) return fail(MK_ERR_ARG, "hidden must be a multiple of 8, <= 8192");
  if (c->vocab <= 0) return fail(MK_ERR_ARG, "vocab must be positive");
  if (!(c->rms_eps > 0.f)) return fail(MK_ERR_ARG, "rms_eps must be positive");
  if (c->ffn <= 0) return fail(MK_ERR_ARG, "ffn must be positive");
  if (c->max_ctx <= 0) return fail(MK_ERR_ARG, "max_ctx must be positive");
  if (c->max_draft < 0 || c->max_draft > 16) return fail(MK_ERR_ARG, "max_draft must be in [0, 16]");
  if (c->weight_format != MK_W_BF16 && c->weight_format != MK_W_Q4K) return fail(MK_ERR_ARG, "unknown weight_format");
  if (c->kv_format != MK_KV_BF16 && c->kv_format != MK_KV_Q8) return fail(MK_ERR_ARG, "unknown kv_format");
  if (c->weight_format == MK_W_Q4K) {
    const long qd = static_cast<long>(c->at_q_heads) * c->at_head_dim;
    if (c->hidden % 256 || c->ffn % 256 || (static_cast<long>(c->dn_heads) * c->dn_dv) % 256 || qd % 256)
      return fail(MK_ERR_ARG, "MK_W_Q4K needs hidden, ffn, dn_heads*dn_dv and at_q_heads*at_head_dim to be multiples of 256");
  }
  const int nd = n_kind(*c, 'D'), na = n_kind(*c, 'A');
  if (nd) {
    if (c->dn_heads <= 0 || c->dn_dk <= 0 || c->dn_dk % 32 || c->dn_dk > 256 || c->dn_dv <= 0 || c->dn_dv > 256)
      return fail(MK_ERR_ARG, "DeltaNet dims: dk must be a multiple of 32 and <= 256, 0 < dv <= 256");
    if (c->conv_width < 2 || c->conv_width > 4) return fail(MK_ERR_ARG, "conv_width must be in [2, 4]");
  }
  if (na) {
    if (c->at_q_heads <= 0 || c->at_kv_heads <= 0 || c->at_q_heads % c->at_kv_heads)
      return fail(MK_ERR_ARG, "attention heads: Hq must be a positive multiple of Hkv");
    if (c->at_q_heads / c->at_kv_heads > 8) return fail(MK_ERR_ARG, "at most 8 query heads per KV head");
    if (c->at_head_dim <= 0 || c->at_head_dim % 64 || c->at_head_dim > 256)
      return fail(MK_ERR_ARG, "at_head_dim must be a multiple of 64, <= 256");
    if (!(c->rope_theta > 0.f)) return fail(MK_ERR_ARG, "rope_theta must be positive");
  }
  return MK_OK;
}

int device_grid(int* grid, int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  int coop = 0;
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, *dev);
  if (!coop) return fail(MK_ERR_RESIDENCY, "device does not support cooperative launches");
  *grid = sms;
  return MK_OK;
}

// Scratch and shared-memory budget checks that depend on the grid size.
bool is_q4(const mk_config& c) { return c.weight_format == MK_W_Q4K; }
size_t q4_rb(size_t cols) { return cols / 256 * mk::kQ4Block; }
// Floats of the input vector the decode kernel stages in shared memory: H, or with Q4
// weights the largest projection input (the out- and down-projections read whole vectors).
int decode_xcap(const mk_config& c) {
  if (!is_q4(c)) return c.hidden;
  const int qd = c.at_q_heads * c.at_head_dim;
  return std::max({c.hidden, c.dn_heads * c.dn_dv, qd, c.ffn});
}

// Whether the decode kernel's shared-memory scratch covers every phase when it keeps
// ltab_entries layer-table entries in shared memory (why: the first shortfall).
bool budget_ok(const mk_config& c, int grid, int ltab_entries, const char** why) {
  auto fail_ = [&](const char* w) {
    *why = w;
    return false;
  };
  const long S = static_cast<long>(mk::decode_scratch_floats(c.hidden, is_q4(c), decode_xcap(c), ltab_entries));
  if (S < 256) return fail_("shared-memory budget exceeded (hidden too large)");
  auto ceil_div = [](long a, long b) { return (a + b - 1) / b; };
  if (n_kind(c, 'D')) {
    const long rows = ceil_div(static_cast<long>(c.dn_heads) * c.dn_dv, grid);
    const long nh = ceil_div(rows, c.dn_dv) + 1;
    if (nh * (2 * c.dn_dk + 2) + 2 * rows > S) return fail_("DeltaNet rows per CTA exceed the scratch budget");
    if (2 * nh * c.dn_dk + rows + nh > 3L * mk::kConsumerThreads)
      return fail_("DeltaNet channels per CTA exceed the prologue budget");
    const long inrows = ceil_div(static_cast<long>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv) + 2 * c.dn_heads, grid);
    if (inrows > mk::kConsumerThreads || 7 * inrows > S)
      return fail_("DeltaNet in-projection rows per CTA exceed the conv budget");
    if (4L * c.dn_heads * 4 + 512 > 4096) return fail_("too many DeltaNet heads for the norm buffer");
  }
  if (n_kind(c, 'A')) {
    const long grp = c.at_q_heads / c.at_kv_heads;
    if (2 * grp * c.at_head_dim + grp * mk::kAttnSub + 3 * grp + 2 * c.at_head_dim > S)
      return fail_("attention scratch budget exceeded");
    const long cols = ceil_div(static_cast<long>(c.at_q_heads) * c.at_head_dim, grid);
    const long nhd = ceil_div(cols, c.at_head_dim) + 1;
    const long ms = mk::decode_max_splits(grid, c.at_kv_heads);
    if (2 * nhd * ms + cols * ms + 2 * cols > S)   // m, l per head and split; the columns' split accumulators
      return fail_("attention columns per CTA exceed the scratch budget");
  }
  if (2 * ceil_div(c.ffn, grid) > S) return fail_("MLP rows per CTA exceed the scratch budget");
  return true;
}

// Valid with the smaller (two-slot) layer table; the whole table is used when it fits too.
int check_budget(const mk_config& c, int grid) {
  const char* why = nullptr;
  return budget_ok(c, grid, 2, &why) ? MK_OK : fail(MK_ERR_ARG, why);
}
bool layer_table_fits(const mk_config& c, int grid) {
  const char* why = nullptr;
  return budget_ok(c, grid, c.n_layers, &why);
}

constexpr int kBatchedPrefillMin = 16;   // shorter prompts run as decode launches

struct Layout {
  mk_sizes sz;
  // packed
  size_t p_table, p_freq, p_embed, p_normf;
  std::vector<size_t> p_layer;   // start of each layer block
  // workspace
  size_t w_sync, w_h, w_z, w_y, w_ob, w_ab, w_part, w_tok, w_g, w_n, w_snap;
  size_t snap_S, snap_conv;
  int max_splits;
  // batched prefill workspace
  int pf_rows;
  size_t pf_h, pf_xhi, pf_xlo, pf_z, pf_y, pf_o, pf_u, pf_w, pf_p, pf_gam, pf_dec, pf_apart, pf_splitk, pf_best;
  size_t pf_kvd = 0;
  size_t pf_vt = 0, pf_img = 0, pf_fq = 0;
  long long pf_nk;
  // batched verify saves
  int vf_rows;
  size_t vf_delta, vf_k, vf_g, vf_raw, vf_logits, vf_greedy, vf_stats;
};

// Tokens per batched prefill pass: the whole context up to 4096 (64 with 4-bit weights,
// whose linear layers run on the CUDA cores per 8-token tile), 0 when a shape is outside
// what the prefill kernels take (then the prompt runs through decode launches).
int prefill_rows(const mk_config& c) {
  const long qd = static_cast<long>(c.at_q_heads) * c.at_head_dim;
  const long kdn = static_cast<long>(c.dn_heads) * c.dn_dv;
  if (c.hidden % 64 || c.ffn % 64 || kdn % 64 || qd % 64) return 0;
  if (c.dn_heads > 64 || c.dn_dk > 128 || c.dn_dv > 128 || c.dn_dv % 16) return 0;
  if (c.at_kv_heads > 0 && c.at_q_heads / c.at_kv_heads > 8) return 0;
  return std::min(c.max_ctx, is_q4(c) ? 64 : 4096);
}

size_t layer_block_bytes(const mk_config& c, char kind) {
  const size_t H = c.hidden, rb = H * 2;
  size_t b = align256(H * 2) * 2;                        // norm1, norm2
  if (is_q4(c)) {
    const size_t rq = q4_rb(H);
    const size_t qd = static_cast<size_t>(c.at_q_heads) * c.at_head_dim;
    if (kind == 'D') {
      const size_t C = static_cast<size_t>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv);
      b += align256((C + 2 * c.dn_heads) * (rq + 16));     // w_in rows + conv-taps tail
      b += align256(C * c.conv_width * 2);                  // conv
      b += align256(H * q4_rb(static_cast<size_t>(c.dn_heads) * c.dn_dv));   // w_out (row-major Q4)
    } else {
      const size_t rows = qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim;
      b += align256(rows * rq);
      b += align256(H * q4_rb(qd));
    }
    b += 2 * align256(static_cast<size_t>(c.ffn) * rq);   // gate, up
    b += align256(H * q4_rb(c.ffn));                      // down (row-major Q4)
    return b;
  }
  if (kind == 'D') {
    const size_t C = static_cast<size_t>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv);
    b += align256((C + 2 * c.dn_heads) * (rb + 16));       // w_in, each row + its conv taps
    b += align256(C * c.conv_width * 2);                    // conv
    b += 2 * align256(static_cast<size_t>(c.dn_heads) * c.dn_dv * rb);   // w_outT, w_out (K-major, prefill)
  } else {
    const size_t qd = static_cast<size_t>(c.at_q_heads) * c.at_head_dim;
    const size_t rows = qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim;
    b += align256(rows * rb);
    b += 2 * align256(qd * rb);                               // w_outT, w_out (K-major, prefill)
  }
  b += 4 * align256(static_cast<size_t>(c.ffn) * rb);     // gate, up, downT, down (K-major, prefill)
  b += align256(2 * static_cast<size_t>(c.ffn) * rb);     // gate / up interleaved by 64 rows (prefill)
  return b;
}

Layout make_layout(const mk_config& c, int grid) {
  Layout L{};
  const size_t H = c.hidden;
  const int nd = n_kind(c, 'D'), na = n_kind(c, 'A');
  size_t off = 0;
  L.p_table = off; off = align256(off + sizeof(mk::LayerW) * c.n_layers);
  L.p_freq = off; off = align256(off + sizeof(double) * (c.at_head_dim > 0 ? c.at_head_dim / 2 : 1));
  L.p_embed = off; off = align256(off + static_cast<size_t>(c.vocab) * (is_q4(c) ? q4_rb(H) : H * 2));
  L.p_normf = off; off = align256(off + H * 2);
  for (int l = 0; l < c.n_layers; ++l) {
    L.p_layer.push_back(off);
    off += layer_block_bytes(c, c.pattern[l]);
  }
  L.sz.packed_bytes = off;

  const size_t C = static_cast<size_t>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv);
  off = 0;
  L.sz.off_S = off; off = align256(off + static_cast<size_t>(nd) * c.dn_heads * c.dn_dv * c.dn_dk * 4);
  L.sz.off_conv = off; off = align256(off + static_cast<size_t>(nd) * c.conv_width * C * 4);
  const size_t kv = static_cast<size_t>(na) * c.at_kv_heads * c.max_ctx * kv_row_bytes(c);
  L.sz.kv_row_bytes = static_cast<int32_t>(kv_row_bytes(c));
  L.sz.off_k = off; off = align256(off + kv);
  L.sz.off_v = off; off = align256(off + kv);
  L.sz.off_pos = off; off = align256(off + 4);
  L.sz.off_err = off; off = align256(off + 4);
  L.sz.state_bytes = off;

  L.max_splits = (na ? mk::decode_max_splits(grid, c.at_kv_heads) : 1);
  off = 0;
  L.w_sync = off; off = align256(off + kResetBytes);   // sync words + per-head norms (zeroed on reset)
  L.w_h = off; off = align256(off + (2 + 3 * mk::kResCopies) * H * 4);   // residual: 2 bases + 3 spread deltas
  const size_t zf = std::max<size_t>(2 * c.dn_heads,
                                     na ? static_cast<size_t>(c.at_q_heads) * c.at_head_dim * (c.at_out_gate ? 2 : 1) +
                                              2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim
                                        : 0);
  L.w_z = off; off = align256(off + zf * 4);
  L.w_y = off; off = align256(off + C * 4);
  L.w_ob = off;
  off = align256(off + std::max<size_t>(static_cast<size_t>(c.dn_heads) * c.dn_dv,
                                        static_cast<size_t>(c.at_q_heads) * c.at_head_dim) * 4 + 16);
  L.w_ab = off; off = align256(off + static_cast<size_t>(c.ffn) * 4);
  L.w_part = off;
  off = align256(off + (na ? static_cast<size_t>(c.at_q_heads) * L.max_splits * (c.at_head_dim + 2) * 4 : 4));
  L.w_tok = off; off = align256(off + (static_cast<size_t>(c.max_ctx) + 8) * 4);
  L.w_g = off; off = align256(off + (static_cast<size_t>(c.max_draft) + 2) * 4);
  L.w_n = off; off = align256(off + 4);
  L.snap_S = static_cast<size_t>(nd) * c.dn_heads * c.dn_dv * c.dn_dk * 4;
  L.snap_conv = static_cast<size_t>(nd) * c.conv_width * C * 4;
  L.w_snap = off;
  if (c.max_draft > 0) off = align256(off + align256(L.snap_S) + align256(L.snap_conv) + 256);
  L.pf_rows = prefill_rows(c);
  if (L.pf_rows > 0) {
    const size_t T = L.pf_rows;
    const size_t qd = static_cast<size_t>(c.at_q_heads) * c.at_head_dim;
    const size_t kdn = static_cast<size_t>(c.dn_heads) * c.dn_dv;
    const size_t at_rows = na ? qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim : 0;
    const size_t kmax = std::max({H, static_cast<size_t>(c.ffn), kdn, qd});
    const size_t zmax = std::max({C + 2 * static_cast<size_t>(c.dn_heads), at_rows, 2 * static_cast<size_t>(c.ffn)});
    const size_t ymax = std::max(C + 2 * static_cast<size_t>(c.dn_heads), qd);
    const size_t omax = std::max(kdn, qd);
    const size_t nch = (T + 63) / 64;
    L.pf_h = off; off = align256(off + T * H * 4);
    L.pf_xhi = off; off = align256(off + T * kmax * 2);
    L.pf_xlo = off; off = align256(off + T * kmax * 2);
    L.pf_z = off; off = align256(off + std::max(T * zmax, static_cast<size_t>(c.vocab)) * 4);   // also the prompt's last logits
    L.pf_y = off; off = align256(off + T * ymax * 4);
    L.pf_o = off; off = align256(off + T * omax * 4);
    L.pf_u = off; off = align256(off + T * kdn * 4);
    L.pf_w = off; off = align256(off + T * static_cast<size_t>(c.dn_heads) * c.dn_dk * 4);
    L.pf_p = off; off = align256(off + nch * c.dn_heads * 64 * 64 * 4);
    L.pf_gam = off; off = align256(off + T * c.dn_heads * 4);
    L.pf_dec = off; off = align256(off + T * c.dn_heads * 4);
    L.pf_apart = off;
    off = align256(off + std::min<size_t>(T, mk::kAttnSplitRows) * c.at_q_heads * mk::kAttnMaxSplit *
                             (static_cast<size_t>(c.at_head_dim) + 2) * 4);
    L.pf_splitk = off; off = align256(off + static_cast<size_t>(mk::kSplitKFloats) * 4);
    L.pf_best = off; off = align256(off + T * 8);
    if (nd > 0 && c.dn_dk == c.dn_dv && (c.dn_dk == 128 || c.dn_dk == 64)) {   // tensor-core chunked delta rule
      const size_t img = 2ull * (c.dn_dk / 64) * 16384 + 16384 + 32768;     // operand images per (chunk, head)
      L.pf_img = off; off = align256(off + nch * c.dn_heads * img);
    }
    // V^T of every kv head of one attention layer for the flash attention: [Hkv][D][nk]
    L.pf_nk = (na && mk::attn_flash_supported(c.at_head_dim)) ? (static_cast<long long>(c.max_ctx) + 63) / 64 * 64 : 0;
    if (L.pf_nk > 0) {
      L.pf_vt = off;
      off = align256(off + static_cast<size_t>(c.at_kv_heads) * c.at_head_dim * static_cast<size_t>(L.pf_nk) * 2);
      L.pf_fq = off;   // the flash kernel's work counter
      off = align256(off + 4);
    }
    if (na && c.kv_format == MK_KV_Q8) {   // one layer's K and V read back as bf16 for the attention kernels
      L.pf_kvd = off;
      off = align256(off + 2ull * c.at_kv_heads * c.max_ctx * c.at_head_dim * 2);
    }
  }
  L.vf_rows = (L.pf_rows > 0 && c.max_draft > 0 && c.max_draft + 1 <= std::min(64, L.pf_rows)) ? c.max_draft + 1 : 0;
  if (L.vf_rows > 0) {
    const size_t R = static_cast<size_t>(L.vf_rows) * nd;
    L.vf_delta = off; off = align256(off + R * c.dn_heads * c.dn_dv * 4);
    L.vf_k = off; off = align256(off + R * c.dn_heads * c.dn_dk * 4);
    L.vf_g = off; off = align256(off + R * c.dn_heads * 4);
    L.vf_raw = off; off = align256(off + R * C * 4);
    L.vf_logits = off; off = align256(off + static_cast<size_t>(L.vf_rows) * c.vocab * 4);
    L.vf_greedy = off; off = align256(off + static_cast<size_t>(L.vf_rows) * 4);
    L.vf_stats = off; off = align256(off + samp_scratch_bytes(L.vf_rows));   // sampled verify
  }
  L.sz.workspace_bytes = off;
  L.sz.grid_ctas = grid;
  L.sz.layer_table_entries = layer_table_fits(c, grid) ? c.n_layers : 2;
  return L;
}

void expected_tensors(const mk_config& c, std::map<std::string, Expect>& ex) {
  const int64_t H = c.hidden;
  auto mat = [&](const std::string& n, int64_t r, int64_t k) {
    if (is_q4(c) && n.find("dn.conv") == std::string::npos)
      ex[n] = Expect{MK_DT_Q4K, 2, {r, k}, static_cast<uint64_t>(r) * static_cast<uint64_t>(q4_rb(static_cast<size_t>(k)))};
    else
      ex[n] = Expect{MK_DT_BF16, 2, {r, k}, static_cast<uint64_t>(r * k * 2)};
  };
  auto vec = [&](const std::string& n, int64_t r) { ex[n] = Expect{MK_DT_BF16, 1, {r, 0}, static_cast<uint64_t>(r * 2)}; };
  mat("embed", c.vocab, H);
  vec("norm_f", H);
  const int64_t C = static_cast<int64_t>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv);
  for (int l = 0; l < c.n_layers; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    vec(p + "norm1", H);
    vec(p + "norm2", H);
    if (c.pattern[l] == 'D') {
      mat(p + "dn.w_in", C + 2 * c.dn_heads, H);
      mat(p + "dn.conv", C, c.conv_width);
      mat(p + "dn.w_out", H, static_cast<int64_t>(c.dn_heads) * c.dn_dv);
    } else {
      const int64_t qd = static_cast<int64_t>(c.at_q_heads) * c.at_head_dim;
      mat(p + "attn.w_in", qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<int64_t>(c.at_kv_heads) * c.at_head_dim, H);
      mat(p + "attn.w_out", H, qd);
    }
    mat(p + "mlp.w_gate", c.ffn, H);
    mat(p + "mlp.w_up", c.ffn, H);
    mat(p + "mlp.w_down", H, c.ffn);
  }
}

std::string shape_str(int ndim, const int64_t* s) {
  std::string r = "[";
  for (int i = 0; i < ndim; ++i) r += (i ? ", " : "") + std::to_string(s[i]);
  return r + "]";
}

int launch_step(mk_model* m, const int32_t* in_tok, int32_t* out_tok, float* logits, cudaStream_t s) {
  mk::DecodeParams p = m->base;
  p.in_token = in_tok;
  p.out_token = out_tok;
  p.logits = logits;
  cudaError_t e = mk::launch_decode(p, m->grid, s);
  if (e == cudaErrorCooperativeLaunchTooLarge)
    return fail(MK_ERR_RESIDENCY, "persistent grid cannot be co-resident: " + std::string(cudaGetErrorString(e)));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  ++m->launches;
  ++m->pos_hint;
  ++m->pos_max;
  return MK_OK;
}

}  // namespace

extern "C" {

int mk_query_sizes(const mk_config* cfg, mk_sizes* out) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!out) return fail(MK_ERR_ARG, "out is NULL");
  int grid = 0, dev = 0;
  rc = device_grid(&grid, &dev);
  if (rc) return rc;
  rc = check_budget(*cfg, grid);
  if (rc) return rc;
  *out = make_layout(*cfg, grid).sz;
  return MK_OK;
}

int mk_load_weights(const mk_config* cfg, const mk_tensor* tensors, int32_t n_tensors, void* d_packed, void* d_state,
                    void* d_workspace, void* stream, mk_model** out) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!out) return fail(MK_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!tensors || n_tensors <= 0) return fail(MK_ERR_ARG, "no tensors given");
  if (!d_packed || !d_state || !d_workspace) return fail(MK_ERR_ARG, "device buffer pointer is NULL");
  const mk_config& c = *cfg;

  // ---- type-check every tensor (host only: nothing here touches the device) ----
  std::map<std::string, Expect> ex;
  expected_tensors(c, ex);
  std::map<std::string, const mk_tensor*> got;
  for (int i = 0; i < n_tensors; ++i) {
    const mk_tensor& t = tensors[i];
    if (!t.name) return fail(MK_ERR_TENSOR, "tensor " + std::to_string(i) + " has no name");
    const std::string nm(t.name);
    auto it = ex.find(nm);
    if (it == ex.end()) return fail(MK_ERR_TENSOR, "unknown tensor '" + nm + "'");
    if (got.count(nm)) return fail(MK_ERR_TENSOR, "tensor '" + nm + "' given twice");
    const Expect& e = it->second;
    if (t.dtype != e.dtype) return fail(MK_ERR_TENSOR, "tensor '" + nm + "': wrong dtype " + std::to_string(t.dtype));
    if (t.ndim != e.ndim) return fail(MK_ERR_TENSOR, "tensor '" + nm + "': wrong rank " + std::to_string(t.ndim));
    for (int d = 0; d < e.ndim; ++d)
      if (t.shape[d] != e.shape[d])
        return fail(MK_ERR_TENSOR, "tensor '" + nm + "': shape " + shape_str(t.ndim, t.shape) + ", expected " +
                                       shape_str(e.ndim, e.shape));
    if (t.bytes != e.bytes) return fail(MK_ERR_TENSOR, "tensor '" + nm + "': wrong byte size");
    if (!t.data) return fail(MK_ERR_TENSOR, "tensor '" + nm + "': data is NULL");
    if (reinterpret_cast<uintptr_t>(t.data) % 16) return fail(MK_ERR_TENSOR, "tensor '" + nm + "': data not 16-byte aligned");
    got[nm] = &t;
  }
  for (auto& kv : ex)
    if (!got.count(kv.first)) return fail(MK_ERR_TENSOR, "missing tensor '" + kv.first + "'");

  int grid = 0, dev = 0;
  rc = device_grid(&grid, &dev);
  if (rc) return rc;
  rc = check_budget(*cfg, grid);
  if (rc) return rc;

  // ---- layout, repack ----
  Layout L = make_layout(c, grid);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* P = static_cast<uint8_t*>(d_packed);
  uint8_t* St = static_cast<uint8_t*>(d_state);
  uint8_t* W = static_cast<uint8_t*>(d_workspace);
  if (reinterpret_cast<uintptr_t>(P) % 256 || reinterpret_cast<uintptr_t>(St) % 256 ||
      reinterpret_cast<uintptr_t>(W) % 256)
    return fail(MK_ERR_ARG, "device buffers must be 256-byte aligned");

  mk_model* m = new mk_model();
  m->cfg = c;
  m->sz = L.sz;
  m->packed = P;
  m->state = St;
  m->ws = W;
  m->grid = grid;
  m->device = dev;
  m->launches = 0;
  m->pos_hint = 0;
  m->pos_max = 0;

  auto copy = [&](const std::string& nm, size_t dst_off) -> cudaError_t {
    const mk_tensor* t = got[nm];
    return cudaMemcpyAsync(P + dst_off, t->data, t->bytes, cudaMemcpyDeviceToDevice, s);
  };
  auto transpose = [&](const std::string& nm, size_t dst_off) -> cudaError_t {
    const mk_tensor* t = got[nm];
    ++m->launches;
    return mk::launch_transpose_bf16(static_cast<const uint16_t*>(t->data), reinterpret_cast<uint16_t*>(P + dst_off),
                                     static_cast<int>(t->shape[0]), static_cast<int>(t->shape[1]), s);
  };
  const size_t H = c.hidden, rb = H * 2;
  const size_t C = static_cast<size_t>(c.dn_heads) * (2 * c.dn_dk + c.dn_dv);
  cudaError_t e = copy("embed", L.p_embed);
  if (e == cudaSuccess) e = copy("norm_f", L.p_normf);
  int di = 0, ai = 0;
  for (int l = 0; l < c.n_layers && e == cudaSuccess && is_q4(c); ++l) {   // Q4_K-style weights
    const std::string p = "layers." + std::to_string(l) + ".";
    size_t off = L.p_layer[l];
    const size_t rq = q4_rb(H);
    mk::LayerW lw{};
    lw.kind = c.pattern[l] == 'D' ? mk::kDeltaNet : mk::kAttention;
    lw.idx = c.pattern[l] == 'D' ? di++ : ai++;
    lw.norm1 = reinterpret_cast<const uint16_t*>(P + off);
    e = copy(p + "norm1", off); off += align256(H * 2);
    lw.norm2 = reinterpret_cast<const uint16_t*>(P + off);
    if (e == cudaSuccess) e = copy(p + "norm2", off);
    off += align256(H * 2);
    if (lw.kind == mk::kDeltaNet) {
      lw.w_in = P + off;
      if (e == cudaSuccess) {
        ++m->launches;
        e = mk::launch_pack_q4_rows_tail(got[p + "dn.w_in"]->data, static_cast<const uint16_t*>(got[p + "dn.conv"]->data),
                                         P + off, static_cast<int>(C + 2 * c.dn_heads), static_cast<int>(rq),
                                         static_cast<int>(C), c.conv_width, s);
      }
      off += align256((C + 2 * c.dn_heads) * (rq + 16));
      lw.conv = reinterpret_cast<const uint16_t*>(P + off);
      if (e == cudaSuccess) e = copy(p + "dn.conv", off);
      off += align256(C * c.conv_width * 2);
      lw.w_out_q4 = P + off;
      if (e == cudaSuccess) e = copy(p + "dn.w_out", off);
      off += align256(H * q4_rb(static_cast<size_t>(c.dn_heads) * c.dn_dv));
    } else {
      const size_t qd = static_cast<size_t>(c.at_q_heads) * c.at_head_dim;
      const size_t rows = qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim;
      lw.w_in = P + off;
      if (e == cudaSuccess) e = copy(p + "attn.w_in", off);
      off += align256(rows * rq);
      lw.w_out_q4 = P + off;
      if (e == cudaSuccess) e = copy(p + "attn.w_out", off);
      off += align256(H * q4_rb(qd));
    }
    lw.w_gate = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_gate", off);
    off += align256(static_cast<size_t>(c.ffn) * rq);
    lw.w_up = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_up", off);
    off += align256(static_cast<size_t>(c.ffn) * rq);
    lw.w_down_q4 = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_down", off);
    m->layers_host.push_back(lw);
    m->pf_layers.push_back(mk_prefill_layer{});
  }
  for (int l = 0; l < c.n_layers && e == cudaSuccess && !is_q4(c); ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    size_t off = L.p_layer[l];
    mk::LayerW lw{};
    mk_prefill_layer pl{};
    lw.kind = c.pattern[l] == 'D' ? mk::kDeltaNet : mk::kAttention;
    lw.idx = c.pattern[l] == 'D' ? di++ : ai++;
    lw.norm1 = reinterpret_cast<const uint16_t*>(P + off);
    e = copy(p + "norm1", off); off += align256(H * 2);
    lw.norm2 = reinterpret_cast<const uint16_t*>(P + off);
    if (e == cudaSuccess) e = copy(p + "norm2", off);
    off += align256(H * 2);
    if (lw.kind == mk::kDeltaNet) {
      lw.w_in = P + off;
      if (e == cudaSuccess) {
        ++m->launches;
        e = mk::launch_pack_rows_tail(static_cast<const uint16_t*>(got[p + "dn.w_in"]->data),
                                      static_cast<const uint16_t*>(got[p + "dn.conv"]->data), P + off,
                                      static_cast<int>(C + 2 * c.dn_heads), static_cast<int>(H), static_cast<int>(C),
                                      c.conv_width, s);
      }
      off += align256((C + 2 * c.dn_heads) * (rb + 16));
      lw.conv = reinterpret_cast<const uint16_t*>(P + off);
      if (e == cudaSuccess) e = copy(p + "dn.conv", off);
      off += align256(C * c.conv_width * 2);
      lw.w_outT = P + off;
      if (e == cudaSuccess) e = transpose(p + "dn.w_out", off);
      off += align256(static_cast<size_t>(c.dn_heads) * c.dn_dv * rb);
      pl.w_out = P + off;
      if (e == cudaSuccess) e = copy(p + "dn.w_out", off);
      off += align256(static_cast<size_t>(c.dn_heads) * c.dn_dv * rb);
    } else {
      const size_t qd = static_cast<size_t>(c.at_q_heads) * c.at_head_dim;
      const size_t rows = qd * (c.at_out_gate ? 2 : 1) + 2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim;
      lw.w_in = P + off;
      if (e == cudaSuccess) e = copy(p + "attn.w_in", off);
      off += align256(rows * rb);
      lw.w_outT = P + off;
      if (e == cudaSuccess) e = transpose(p + "attn.w_out", off);
      off += align256(qd * rb);
      pl.w_out = P + off;
      if (e == cudaSuccess) e = copy(p + "attn.w_out", off);
      off += align256(qd * rb);
    }
    lw.w_gate = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_gate", off);
    off += align256(static_cast<size_t>(c.ffn) * rb);
    lw.w_up = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_up", off);
    off += align256(static_cast<size_t>(c.ffn) * rb);
    lw.w_downT = P + off;
    if (e == cudaSuccess) e = transpose(p + "mlp.w_down", off);
    off += align256(static_cast<size_t>(c.ffn) * rb);
    pl.w_down = P + off;
    if (e == cudaSuccess) e = copy(p + "mlp.w_down", off);
    off += align256(static_cast<size_t>(c.ffn) * rb);
    pl.w_gu = P + off;   // rows 128 b .. + 63: gate rows 64 b ..; rows 128 b + 64 .. + 127: up rows 64 b ..
    if (e == cudaSuccess && c.ffn % 64 == 0) {
      const size_t blk = 64 * rb;
      e = cudaMemcpy2DAsync(P + off, 2 * blk, got[p + "mlp.w_gate"]->data, blk, blk, c.ffn / 64,
                            cudaMemcpyDeviceToDevice, s);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(P + off + blk, 2 * blk, got[p + "mlp.w_up"]->data, blk, blk, c.ffn / 64,
                              cudaMemcpyDeviceToDevice, s);
    }
    m->layers_host.push_back(lw);
    m->pf_layers.push_back(pl);
  }
  std::vector<double> freq(c.at_head_dim > 0 ? c.at_head_dim / 2 : 1, 0.0);
  for (int i = 0; i < c.at_head_dim / 2; ++i)
    freq[i] = std::pow(static_cast<double>(c.rope_theta), -2.0 * i / static_cast<double>(c.at_head_dim));
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(P + L.p_table, m->layers_host.data(), sizeof(mk::LayerW) * c.n_layers, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(P + L.p_freq, freq.data(), sizeof(double) * freq.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(St, 0, L.sz.state_bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(W, 0, L.sz.workspace_bytes, s);
  // the two host vectors above are pageable: make sure the copies have read them
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    delete m;
    return cuda_fail(e, "weight repack");
  }

  mk::DecodeParams& b = m->base;
  b = mk::DecodeParams{};
  b.layers = reinterpret_cast<const mk::LayerW*>(P + L.p_table);
  b.n_layers = c.n_layers;
  b.embed = P + L.p_embed;
  b.norm_f = reinterpret_cast<const uint16_t*>(P + L.p_normf);
  b.inv_freq = reinterpret_cast<const double*>(P + L.p_freq);
  b.H = c.hidden; b.V = c.vocab; b.F = c.ffn;
  b.Hd = c.dn_heads; b.dk = c.dn_dk; b.dv = c.dn_dv; b.convw = c.conv_width; b.C = static_cast<int>(C);
  b.Hq = c.at_q_heads; b.Hkv = c.at_kv_heads; b.D = c.at_head_dim; b.gated = c.at_out_gate;
  b.at_in_rows = static_cast<int>(static_cast<size_t>(c.at_q_heads) * c.at_head_dim * (c.at_out_gate ? 2 : 1) +
                                  2 * static_cast<size_t>(c.at_kv_heads) * c.at_head_dim);
  b.max_ctx = c.max_ctx;
  b.row_bytes = static_cast<int>(is_q4(c) ? q4_rb(H) : rb);
  b.q4 = is_q4(c) ? 1 : 0;
  b.ltab_full = layer_table_fits(c, grid) ? 1 : 0;
  b.rb_dn_out = static_cast<int>(q4_rb(static_cast<size_t>(c.dn_heads) * c.dn_dv));
  b.rb_at_out = static_cast<int>(q4_rb(static_cast<size_t>(c.at_q_heads) * c.at_head_dim));
  b.rb_ffn = static_cast<int>(q4_rb(c.ffn));
  b.xcap = decode_xcap(c);
  b.obuf = reinterpret_cast<float*>(W + L.w_ob);
  b.abuf = reinterpret_cast<float*>(W + L.w_ab);
  b.eps = c.rms_eps;
  b.S = reinterpret_cast<float*>(St + L.sz.off_S);
  b.conv_ring = reinterpret_cast<float*>(St + L.sz.off_conv);
  b.kc = reinterpret_cast<uint16_t*>(St + L.sz.off_k);
  b.vc = reinterpret_cast<uint16_t*>(St + L.sz.off_v);
  b.kv_q8 = c.kv_format == MK_KV_Q8 ? 1 : 0;
  b.kv_rb = static_cast<int>(kv_row_bytes(c));
  b.pos = reinterpret_cast<int*>(St + L.sz.off_pos);
  b.err = reinterpret_cast<int*>(St + L.sz.off_err);
  b.hbuf = reinterpret_cast<float*>(W + L.w_h);
  b.z = reinterpret_cast<float*>(W + L.w_z);
  b.part = reinterpret_cast<float*>(W + L.w_part);
  b.bar = reinterpret_cast<unsigned*>(W + L.w_sync);
  b.done = reinterpret_cast<unsigned*>(W + L.w_sync + 128);
  b.amax = reinterpret_cast<unsigned long long*>(W + L.w_sync + 256);
  b.ssq = reinterpret_cast<float*>(W + L.w_sync + 512);
  b.ybuf = reinterpret_cast<float*>(W + L.w_y);
  b.max_splits = L.max_splits;
  m->ws_tok = reinterpret_cast<int32_t*>(W + L.w_tok);
  m->ws_g = reinterpret_cast<int32_t*>(W + L.w_g);
  m->ws_n = reinterpret_cast<int32_t*>(W + L.w_n);
  m->ws_snap = c.max_draft > 0 ? W + L.w_snap : nullptr;
  m->snap_S_bytes = L.snap_S;
  m->step_scratch_bytes = L.w_tok;   // sync words, residual, projections, attention partials
  m->snap_conv_bytes = L.snap_conv;
  m->pf.rows = L.pf_rows;
  if (L.pf_rows > 0) {
    m->pf.h = reinterpret_cast<float*>(W + L.pf_h);
    m->pf.xhi = reinterpret_cast<uint16_t*>(W + L.pf_xhi);
    m->pf.xlo = reinterpret_cast<uint16_t*>(W + L.pf_xlo);
    m->pf.z = reinterpret_cast<float*>(W + L.pf_z);
    m->pf.y = reinterpret_cast<float*>(W + L.pf_y);
    m->pf.o = reinterpret_cast<float*>(W + L.pf_o);
    m->pf.u = reinterpret_cast<float*>(W + L.pf_u);
    m->pf.w = reinterpret_cast<float*>(W + L.pf_w);
    m->pf.p = reinterpret_cast<float*>(W + L.pf_p);
    m->pf.gam = reinterpret_cast<float*>(W + L.pf_gam);
    m->pf.dec = reinterpret_cast<float*>(W + L.pf_dec);
    m->pf.apart = reinterpret_cast<float*>(W + L.pf_apart);
    m->pf.splitk = reinterpret_cast<float*>(W + L.pf_splitk);
    m->pf.best = reinterpret_cast<unsigned long long*>(W + L.pf_best);
    m->pf.nk_max = L.pf_nk;
    m->pf.kvd = L.pf_kvd ? reinterpret_cast<uint16_t*>(W + L.pf_kvd) : nullptr;
    if (L.pf_img) m->pf.img = W + L.pf_img;
    if (L.pf_nk > 0) {
      m->pf.vt = reinterpret_cast<uint16_t*>(W + L.pf_vt);
      m->pf.flash_items = reinterpret_cast<int*>(W + L.pf_fq);
    }
  }
  m->vf.rows = L.vf_rows;
  if (L.vf_rows > 0) {
    m->vf.delta = reinterpret_cast<float*>(W + L.vf_delta);
    m->vf.k = reinterpret_cast<float*>(W + L.vf_k);
    m->vf.g = reinterpret_cast<float*>(W + L.vf_g);
    m->vf.raw = reinterpret_cast<float*>(W + L.vf_raw);
    m->vf.logits = reinterpret_cast<float*>(W + L.vf_logits);
    m->vf.greedy = reinterpret_cast<int32_t*>(W + L.vf_greedy);
    m->vf.stats = reinterpret_cast<double*>(W + L.vf_stats);
  }
  *out = m;
  return MK_OK;
}

int mk_reset_state(mk_model* m, void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(m->state, 0, m->sz.state_bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(m->ws, 0, kResetBytes, s);   // sync words and per-head norms
  if (e != cudaSuccess) return cuda_fail(e, "reset");
  m->pos_hint = 0;
  m->pos_max = 0;
  return MK_OK;
}

int mk_set_position(mk_model* m, int32_t pos, void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (pos < 0 || pos > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "position outside [0, max_ctx]");
  mk::set_int_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(m->base.pos, pos);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "set position");
  ++m->launches;
  m->pos_hint = pos;
  m->pos_max = pos;
  return MK_OK;
}

int mk_decode_step(mk_model* m, const int32_t* d_in_token, int32_t* d_out_token, float* d_logits, void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!d_in_token || !d_out_token) return fail(MK_ERR_ARG, "token pointer is NULL");
  if (m->pos_hint + 1 > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "context capacity reached");
  return launch_step(m, d_in_token, d_out_token, d_logits, static_cast<cudaStream_t>(stream));
}

int mk_prefill(mk_model* m, const int32_t* d_tokens, int32_t n, float* d_last_logits, int32_t* d_next_token,
               void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!d_tokens || n <= 0) return fail(MK_ERR_ARG, "no prompt tokens");
  if (m->pos_hint + n > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "prompt exceeds the context capacity");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* sink = m->ws_tok + m->cfg.max_ctx + 4;
  if (m->pf.rows > 0 && n > kBatchedPrefillMin) {
    // every token through the batched layers, then the last token's logits and greedy token
    // from its residual row (final norm, LM head over one row, argmax)
    int rc = mk_prefill_batched(m, d_tokens, n, s);
    if (rc) return rc;
    return mk_prefill_tail(m, n, d_last_logits, d_next_token, s);
  }
  for (int i = 0; i < n; ++i) {
    const bool last = (i == n - 1);
    int rc = launch_step(m, d_tokens + i, last && d_next_token ? d_next_token : sink, last ? d_last_logits : nullptr, s);
    if (rc) return rc;
  }
  return MK_OK;
}

int mk_verify_drafts(mk_model* m, const int32_t* d_tokens, int32_t K, int32_t* d_n_accepted, int32_t* d_out_tokens,
                     float* d_logits, void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!d_tokens || !d_n_accepted || !d_out_tokens) return fail(MK_ERR_ARG, "pointer is NULL");
  if (K < 1 || K > m->cfg.max_draft) return fail(MK_ERR_ARG, "K outside [1, max_draft]");
  if (m->pos_hint + K + 1 > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "drafts exceed the context capacity");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m->vf.rows >= K + 1)
    return mk_verify_batched(m, d_tokens, K, d_n_accepted, d_out_tokens, d_logits, s);
  const mk::DecodeParams& b = m->base;
  uint8_t* snapS = m->ws_snap;
  uint8_t* snapC = snapS + align256(m->snap_S_bytes);
  uint8_t* snapP = snapC + align256(m->snap_conv_bytes);
  // 1. snapshot the recurrent state (S, conv history, position)
  cudaError_t e = cudaMemcpyAsync(snapS, b.S, m->snap_S_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(snapC, b.conv_ring, m->snap_conv_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(snapP, b.pos, 4, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "verify snapshot");
  const int64_t pos0 = m->pos_hint;
  // 2. score the K + 1 positions
  for (int i = 0; i <= K; ++i) {
    int rc = launch_step(m, d_tokens + i, m->ws_g + i,
                         d_logits ? d_logits + static_cast<size_t>(i) * m->cfg.vocab : nullptr, s);
    if (rc) return rc;
  }
  // 3. longest matching prefix + bonus token
  mk::accept_kernel<<<1, 32, 0, s>>>(d_tokens, m->ws_g, K, m->ws_n, d_n_accepted, d_out_tokens);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "accept");
  ++m->launches;
  // 4. roll back and 5. replay the accepted prefix (steps past n return at once)
  e = cudaMemcpyAsync(b.S, snapS, m->snap_S_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(b.conv_ring, snapC, m->snap_conv_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(b.pos, snapP, 4, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "verify rollback");
  m->pos_hint = pos0;
  for (int i = 0; i <= K; ++i) {
    mk::DecodeParams p = m->base;
    p.in_token = d_tokens + i;
    p.out_token = m->ws_tok + m->cfg.max_ctx + 4;
    p.logits = nullptr;
    p.gate_n = m->ws_n;
    p.gate_i = i;
    e = mk::launch_decode(p, m->grid, s);
    if (e != cudaSuccess) return cuda_fail(e, "verify replay");
    ++m->launches;
  }
  m->pos_hint = pos0 + 1;   // at least one position is always committed; the exact count is on the device
  m->pos_max = pos0 + K + 1;
  return MK_OK;
}

int mk_verify_drafts_sampled(mk_model* m, const int32_t* d_tokens, int32_t K, float temperature,
                             const float* d_uniforms, int32_t* d_n_accepted, int32_t* d_out_tokens, float* d_logits,
                             void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!d_tokens || !d_uniforms || !d_n_accepted || !d_out_tokens) return fail(MK_ERR_ARG, "pointer is NULL");
  if (K < 1 || K > m->cfg.max_draft) return fail(MK_ERR_ARG, "K outside [1, max_draft]");
  if (!(temperature > 0.0f) || !std::isfinite(temperature))
    return fail(MK_ERR_ARG, "temperature must be positive and finite");
  if (m->pos_hint + K + 1 > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "drafts exceed the context capacity");
  if (m->vf.rows < K + 1)
    return fail(MK_ERR_CAPACITY, "sampled verify needs the batched verify workspace (max_draft + 1 <= 64)");
  return mk_verify_batched(m, d_tokens, K, d_n_accepted, d_out_tokens, d_logits, static_cast<cudaStream_t>(stream),
                           temperature, d_uniforms);
}

int mk_generate(mk_model* m, const int32_t* h_prompt, int32_t n_prompt, int32_t* h_out, int32_t n_new, void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!h_prompt || n_prompt <= 0 || !h_out || n_new <= 0) return fail(MK_ERR_ARG, "bad prompt or output buffer");
  if (m->pos_hint + n_prompt + n_new - 1 > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "generation exceeds max_ctx");
  if (n_prompt + n_new > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "generation exceeds max_ctx");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* d_prompt = m->ws_tok;
  int32_t* d_gen = m->ws_tok + n_prompt;
  cudaError_t e = cudaMemcpyAsync(d_prompt, h_prompt, sizeof(int32_t) * n_prompt, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "prompt upload");
  int rc = mk_prefill(m, d_prompt, n_prompt, nullptr, d_gen, stream);
  if (rc) return rc;
  for (int i = 1; i < n_new; ++i) {
    rc = launch_step(m, d_gen + i - 1, d_gen + i, nullptr, s);
    if (rc) return rc;
  }
  e = cudaMemcpyAsync(h_out, d_gen, sizeof(int32_t) * n_new, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "generate");
  return MK_OK;
}

int mk_sync_status(mk_model* m, void* stream, int32_t* dev_err) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&word, m->base.err, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "sync");
  if (dev_err) *dev_err = word;
  if (word) {
    char buf[96];
    snprintf(buf, sizeof buf, "device error word 0x%x", word);
    return fail(MK_ERR_DEVICE, buf);
  }
  return MK_OK;
}

int mk_phase_trace(mk_model* m, uint64_t* d_trace, int32_t capacity) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (d_trace && capacity <= 0) return fail(MK_ERR_ARG, "capacity must be positive");
  m->base.trace = reinterpret_cast<unsigned long long*>(d_trace);
  m->base.trace_cap = d_trace ? capacity : 0;
  return MK_OK;
}

int64_t mk_launch_count(const mk_model* m) { return m ? m->launches : 0; }

const char* mk_last_error(void) { return g_err.c_str(); }

void mk_free(mk_model* m) { delete m; }

}  // extern "C"
