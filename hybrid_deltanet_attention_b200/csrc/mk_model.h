// Host-side model handle of libmk.so (internal; the C ABI only sees an opaque pointer).
#pragma once
#include <cstdint>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

#include <string>

// Sets the thread-local message returned by mk_last_error().
void mk_set_last_error(const std::string& msg);

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
  int64_t pos_hint;      // host shadow of the device position (calls through this handle)
  // workspace sub-buffers used by the host-side drivers
  int32_t* ws_tok;       // [max_ctx + 8] token staging for prefill / generate
  int32_t* ws_g;         // [max_draft + 1] greedy tokens of a verify pass
  int32_t* ws_n;         // accepted-draft count of the last verify pass
  uint8_t* ws_snap;      // DeltaNet S + conv history + pos snapshot for verify
  size_t snap_S_bytes, snap_conv_bytes;
  size_t step_scratch_bytes;   // leading part of the workspace one decode step uses
};
