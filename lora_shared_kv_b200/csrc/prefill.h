// Internal interface of the prefill-chunk kernel.
#pragma once

#include "lrkv_internal.h"

namespace lrkv {

struct PrefillParams {
  const void* q;             // [N, T, Hq, d] bf16, contiguous
  const int32_t* offsets;    // [N] or null
  const int32_t* page_table; // null => dense
  long long pt_stride;
  int num_pages;
  void* out;                 // [N, T, Hq, d]
  int out_f32;
  int N, Hq, Hkv, G;
  int T, L0, session;
  int mode;
  int n_tb;                  // 128-row tiles per (KV head, agent)
  float scale_log2;
  unsigned* flags;
};

// Four CUtensorMap objects, in order: K, V, U, B.
struct PrefillMaps {
  const void* maps;
};

int prefill_smem_bytes(int D, int RK);
lrkv_status launch_prefill(const PrefillParams& p, const PrefillMaps& m, int D, int RK, int grid, void* stream);

}  // namespace lrkv
