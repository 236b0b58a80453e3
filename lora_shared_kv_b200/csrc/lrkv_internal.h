// Internal definitions shared by the C-ABI layer and the kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/lrkv.h"

// Device-side flag bits, kept in the first word of every workspace.
#define LRKV_DEVFLAG_SEQLEN 0x1u    // a seq_len outside [0, max_seq_len] or past the U capacity
#define LRKV_DEVFLAG_OFFSET 0x2u    // a negative aLoRA offset (treated as 0)
#define LRKV_DEVFLAG_PAGE 0x4u      // a page id outside [0, num_pages) (tile skipped)
#define LRKV_DEVFLAG_TIMEOUT 0x8u   // a bounded wait gave up

namespace lrkv {

constexpr int kWsHeaderBytes = 256;     // flags word + padding at the start of a workspace
constexpr int kKeysPerTile = 64;        // keys per K/V tile (one TMA box, one page)
constexpr int kMaxRowsPerItem = 32;     // query rows (agents x GQA heads) per decode work item
constexpr int kMaxAgents = 16;
constexpr int kTileRun = 4;             // decode tiles visited contiguously (see TileOrder in decode.cu)
constexpr int kWholeItemSlackTiles = 12;  // decode: whole items per CTA if that adds at most this many tiles

// Spin cap of every bounded wait.  A try_wait suspends for a short while per
// attempt, so this is well over a second of waiting: far beyond any healthy
// pipeline stall, and the kernel then records LRKV_DEVFLAG_TIMEOUT and returns.
constexpr uint32_t kSpinCap = 1u << 24;

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------
struct DecodeParams {
  const void* q;             // bf16 [S, N, Hq, d]
  const void* b;             // bf16 [N, r, Hkv*d]
  const int32_t* seq_lens;   // [S]
  const int32_t* offsets;    // [S, N] or null
  const int32_t* page_table; // null => dense
  long long pt_stride;
  void* out;
  int out_f32;
  int S, N, Hq, Hkv, G;      // Hkv: KV heads of this launch (the K/V view's heads)
  int g_base, Hkv_total;     // global index of the view's head 0; KV heads of the model (q, out, B)
  int rows_total;            // N * G
  int rows_per_group;        // rows of one work item (<= 32)
  int n_rg;                  // row groups per (session, KV head)
  int n_u_slots;             // U tiles staged per K/V tile
  int mode;
  int max_seq_len;
  int u_rows;
  int num_pages;
  int paged;
  int nt;                    // key tiles per work item
  int tile_stride;           // runs of kTileRun tiles of an item are visited in the order (j * tile_stride) mod runs
  int items;                 // S * Hkv * n_rg
  long long W;               // items * nt (flattened tile count)
  int max_segs;              // partial slots per item
  int stages;
  float scale_log2;          // softmax_scale * log2(e)
  float* partials;
  int* tickets;
  unsigned* flags;
  // Failure-detection test hook (lrkv_debug_stall_next_launch): every bounded
  // wait gives up after spin_cap failed attempts, and with `stall` the
  // producer issues no copies, so the consumers' waits run out.
  unsigned spin_cap;
  int stall;
};

// Consumer warp groups of the decode kernel (NT warps each, eight query rows
// per warp).  Tile n of a CTA goes to group n % groups and to ring stage
// n % stages.  More groups keep more tiles in flight per SM; three fit the
// register file for up to 16 rows per item (NT <= 2), two for 24.  Items of
// up to 8 rows that are split over CTAs take four (measured on Qwen3 shapes
// with 128 items: 8192 keys, split over 148 CTAs, 2.428 -> 2.329 ms per 28
// layers); whole items keep three (1024 / 2048 / 4096 keys, one item per CTA,
// 1.7 / 3.7 / 4.5% slower with four: a group holds its ring stage while it
// computes, and those launches need more stages loading per SM).
__host__ __device__ constexpr int decode_groups(int NT, bool split) {
  return NT == 1 && split ? 4 : (NT <= 2 ? 3 : 2);
}

// Shared-memory plan of the decode kernel (bytes from a 1024-aligned base).
struct DecodeSmem {
  int stage_bytes, ring_bytes, merge_off, scw_off, a_off, bar_off, total;
};

__host__ __device__ inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

__host__ __device__ inline DecodeSmem decode_smem_plan(int D, int NT, int RK, int n_u_slots, int stages) {
  DecodeSmem s;
  const int RP = NT * 8;
  s.stage_bytes = round_up(2 * kKeysPerTile * D * 2 + n_u_slots * kKeysPerTile * RK * 2, 1024);
  s.ring_bytes = stages * s.stage_bytes;
  s.merge_off = s.ring_bytes;
  const int rec = RP * (D + RK + 2) * 4;
  s.scw_off = s.merge_off + 2 * rec;      // two records: segments alternate
  s.a_off = s.scw_off + 2 * 8 * RP * 4;   // scale tables of the consumers and of the epilogue warp
  s.bar_off = round_up(s.a_off + kMaxAgents * 4, 16);
  s.total = s.bar_off + (2 * stages + 4) * 8 + stages * 4 + 64;
  return s;
}

inline size_t decode_record_floats(int NT, int D, int RK) { return (size_t)NT * 8 * (D + RK + 2); }

// Owner CTA of flattened tile t when W tiles are split evenly over C CTAs:
// CTA c covers [c*W/C, (c+1)*W/C).
__host__ __device__ inline long long owner_cta(long long t, long long W, long long C) {
  return ((t + 1) * C - 1) / W;
}

// Value projection [V_base | U_1 .. U_n] = X [W0_v | A_1 .. A_n] into the caches.
struct VprojParams {
  int T, Dm, Hkv, d, n_u, r, ncols;  // ncols = Hkv d + n_u r
  int start_row, session;
  uint16_t* v;                       // base value cache (bf16)
  long long v_ss, v_sh, v_st, v_sp;  // strides (elements): session, head, token, page
  const int32_t* page_table;         // null => dense
  long long pt_stride;
  int page_size, num_pages;
  uint16_t* u;                       // low-rank caches (bf16)
  long long u_ss, u_sa, u_st;
  unsigned* flags;                   // device status word
};

// ---------------------------------------------------------------------------
// launchers (defined in the kernel translation units)
// ---------------------------------------------------------------------------
struct TmaMaps;  // opaque; holds CUtensorMap objects

lrkv_status launch_decode(const DecodeParams& p, int D, int NT, int RK, int groups, const void* tmK, const void* tmV,
                          const void* tmU, int smem_bytes, int ctas, void* stream);
int decode_max_smem_optin();
int vproj_smem_bytes();
lrkv_status launch_vproj(const VprojParams& p, const void* tmX, const void* tmW, int sms, void* stream);

lrkv_status launch_append(const void* x, const void* a, int n_a, const int* row_begin, const int* row_end,
                          int u_shift, int Dm, int r, void* u, long long u_ss, long long u_sa, long long u_st,
                          int session, void* stream);

}  // namespace lrkv
