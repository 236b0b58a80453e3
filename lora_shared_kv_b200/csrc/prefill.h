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
  // stream-K split of the (tile, 128-key block) pairs over the CTAs
  long long W_ga;            // blocks of the n_tb tiles of one (KV head, agent)
  long long W;               // blocks in all
  int max_parts;             // CTAs that can share one tile
  int* tickets;              // [tiles], zero between launches
  float* partials;           // [tiles][max_parts][128 rows: m, l, O + Z B (d)]
  unsigned spin_cap;         // failed attempts after which a bounded wait gives up
  int stall;                 // test hook: the producers issue no copies (the waits run out)
};

// Stream-K plan of a prefill launch and its workspace (bytes from the start of
// the workspace: the status header, tickets, partial records).
struct PrefillPlan {
  int n_tb, tiles, ctas, max_parts;
  long long W_ga, W;
  size_t tickets_off, partials_off, bytes;
};
PrefillPlan plan_prefill(int T, int L0, int G, int Hkv, int N, int D, int sms);

// Four CUtensorMap objects, in order: K, V, U, B.
struct PrefillMaps {
  const void* maps;
};

int prefill_smem_bytes(int D, int RK);
lrkv_status launch_prefill(const PrefillParams& p, const PrefillMaps& m, int D, int RK, int grid, void* stream);

}  // namespace lrkv
