// Split-K decode attention over a shared base K/V cache with per-agent
// low-rank value caches.
//
// Computes, for every (session s, agent i, query head h), with g = h / G:
//     o = ( P V_base,g  +  (P Umask_i) B_i,g ) / l,   P = exp(q K_base,g^T * scale - m)
// which is Eq. 12 of "LRAgent: Efficient KV Cache Sharing for Multi-LoRA LLM
// Agents" (Pith review, "What carries the argument"): the attention-weighted
// rank-r values P U_i are accumulated first (Z, r floats per query row, in
// registers) and the up-projection B_i is applied once per row at the end, so
// the L x d adapter cache is never formed.  Umask_i drops the rows before the
// agent's aLoRA activation offset ("RoleKV", "What it does").
//
// Design (B200, sm_100a):
//  * One work item = (session, KV head, row group).  Its rows are all the
//    query rows that read this KV head: every agent x every GQA head, so each
//    K/V tile is read from HBM once for all agents.
//  * The flattened (item, key tile) space is split evenly over one CTA per SM
//    (stream-K style); an item cut by a CTA boundary is merged by the last CTA
//    to finish it (atomic ticket), which also applies Z B_i and the 1/l.  When
//    the items fit one per SM and that adds only a few tiles to a CTA's share,
//    the host gives each CTA one whole item instead (nothing to merge).
//  * A producer warp moves 64-key K/V tiles (128B-swizzled) and the rank-r U
//    tiles with the Tensor Memory Accelerator into a ring of stages guarded by
//    mbarriers.  U tiles wholly before an agent's offset are never loaded.
//  * Consumer warps come in owner groups (three when an item has at most 16
//    rows, two for 24) that take a CTA's tiles round-robin; a warp owns 8
//    query rows over all 64 keys of its group's tiles and runs the
//    contractions on the tensor cores with keys as the M dimension
//    (S^T = K Q^T, O^T += V^T P^T, Z^T += U_i^T P^T), so a handful of query
//    rows pads only to a multiple of 8.  The score accumulators are re-laid
//    into the P^T operand with movmatrix; the row max takes warp shuffles.
//    Rows past seq_len and U rows before a_i are removed by selects on the
//    operands, never by multiplying with 0.  The groups merge their rows at
//    the end of a CTA's segment of an item.
//  * An epilogue warp publishes (or, as the item's last CTA, combines and
//    finishes) every segment but the CTA's last while the consumers stream
//    on; the consumers finish the last one themselves.
#include <float.h>
#include <math.h>

#include "common.cuh"

namespace lrkv {

namespace {

constexpr int KT = kKeysPerTile;
constexpr int SEG_CHUNK = 8;               // partial records combined per pass

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  uintptr_t v = reinterpret_cast<uintptr_t>(p);
  return reinterpret_cast<uint8_t*>((v + 1023) & ~uintptr_t(1023));
}

// Per-segment facts both roles derive identically.
struct Seg {
  int item, s, g, rg;
  int lo, hi;        // key tiles [lo, hi) of this CTA on this item, clipped to the session's length
  int sl;            // session length (clamped)
  int row_lo, rows;  // query rows [row_lo, row_lo + rows) of the N*G rows of this KV head
  int i_lo, n_ag;    // agents spanned by the rows
};

__device__ __forceinline__ Seg make_seg(const DecodeParams& p, long long t, long long t_end, bool flag_errors) {
  Seg sg;
  sg.item = (int)(t / p.nt);
  sg.lo = (int)(t - (long long)sg.item * p.nt);
  long long hi = t_end - (long long)sg.item * p.nt;
  sg.hi = hi < p.nt ? (int)hi : p.nt;
  sg.rg = sg.item % p.n_rg;
  const int sh = sg.item / p.n_rg;
  sg.g = sh % p.Hkv;
  sg.s = sh / p.Hkv;
  int sl = __ldg(p.seq_lens + sg.s);
  if (sl < 0 || sl > p.max_seq_len || sl > p.u_rows) {
    if (flag_errors) atomicOr(p.flags, LRKV_DEVFLAG_SEQLEN);
    sl = sl < 0 ? 0 : sl;
    sl = sl > p.max_seq_len ? p.max_seq_len : sl;
    sl = sl > p.u_rows ? p.u_rows : sl;
  }
  sg.sl = sl;
  return sg;
}

__device__ __forceinline__ void seg_rows(const DecodeParams& p, Seg& sg) {
  sg.row_lo = sg.rg * p.rows_per_group;
  int row_hi = sg.row_lo + p.rows_per_group;
  row_hi = row_hi < p.rows_total ? row_hi : p.rows_total;
  sg.rows = row_hi - sg.row_lo;
  sg.i_lo = sg.row_lo / p.G;
  sg.n_ag = (row_hi - 1) / p.G - sg.i_lo + 1;
}

__device__ __forceinline__ int seg_tiles_valid(const Seg& sg) { return (sg.sl + KT - 1) / KT; }

// Visiting order of an item's tiles.  Tiles go in runs of kTileRun
// (contiguous in HBM); the full runs are visited in the order
// (j * stride) mod runs with a stride coprime to the run count (near 0.618 of
// it), and a partial last run stays in place.  Every contiguous range of k then
// covers the item evenly, so the tiles past the agents' offsets (which carry
// the low-rank work) spread evenly over the CTAs that share an item.  The
// softmax result does not depend on the order.  The iterator steps with one
// add and one compare; the modulo runs once per segment.
struct TileOrder {
  int runs, stride, r, w;
  __device__ __forceinline__ void start(const DecodeParams& p, int k0) {
    runs = p.nt / kTileRun;
    stride = p.tile_stride;
    const int j = k0 / kTileRun;
    w = k0 % kTileRun;
    r = j < runs ? (int)(((long long)j * stride) % runs) : -1 - j;
  }
  __device__ __forceinline__ int tile() const { return r >= 0 ? r * kTileRun + w : (-1 - r) * kTileRun + w; }
  __device__ __forceinline__ void next() {
    if (++w == kTileRun) {
      w = 0;
      if (r >= 0) {
        ++run_index;
        if (run_index < runs) {
          r += stride;
          if (r >= runs) r -= runs;
        } else {
          r = -1 - run_index;
        }
      } else {
        --r;
      }
    }
  }
  int run_index;
};

__device__ __forceinline__ TileOrder tile_order(const DecodeParams& p, int k0) {
  TileOrder o;
  o.start(p, k0);
  o.run_index = k0 / kTileRun;
  return o;
}

__device__ __forceinline__ int load_offset(const DecodeParams& p, int s, int agent, bool flag_errors) {
  if (p.offsets == nullptr) return 0;
  int a = __ldg(p.offsets + (size_t)s * p.N + agent);
  if (a < 0) {
    if (flag_errors) atomicOr(p.flags, LRKV_DEVFLAG_OFFSET);
    a = 0;
  }
  return a;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float(((uint32_t)v) << 16); }

// ---------------------------------------------------------------------------
// producer warp
// ---------------------------------------------------------------------------
// Tile n of the CTA (counted over all its segments) goes to ring stage
// n % stages.  Before copying, the producer writes n into seq[stage]; a
// consumer waits for its tile number there before it waits on the stage's
// mbarrier, so that a parity wait can never be satisfied by an older phase
// of the same stage (the stage count need not be a multiple of the number
// of consumer groups).
template <int D, int RK>
__device__ void decode_producer(const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                const CUtensorMap* tmU, uint8_t* ring, int stage_bytes, uint64_t* full,
                                uint64_t* empty, volatile int* seq, volatile int* abort_flag, long long t_begin,
                                long long t_end) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = policy_evict_first();
  const uint64_t pol_u = policy_evict_last();
  constexpr int KV_BYTES = KT * D * 2;
  constexpr int U_BYTES = KT * RK * 2;
  int stage = 0;
  uint32_t phase = 0;
  int n = 0;
  bool stop = p.stall != 0;  // the test hook: issue nothing, so the consumers' waits run out
  for (long long t = t_begin; t < t_end && !stop;) {
    Seg sg = make_seg(p, t, t_end, false);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    const int nts = seg_tiles_valid(sg);
    // lane j < n_ag holds the offset of agent i_lo + j
    const int my_a = lane < sg.n_ag ? load_offset(p, sg.s, sg.i_lo + lane, false) : 0x7fffffff;
    int pid_reg = 0;
    TileOrder ord = tile_order(p, sg.lo);
    for (int kk = sg.lo; kk < sg.hi; ++kk, ord.next()) {
      const int tile = ord.tile();
      const int k = kk - sg.lo;
      if (p.paged && (k & 31) == 0) {  // page ids of the next 32 tiles, one per lane
        const int k2 = kk + lane;
        const int t2 = k2 < sg.hi ? tile_order(p, k2).tile() : nts;
        pid_reg = t2 < nts ? __ldg(p.page_table + (size_t)sg.s * p.pt_stride + t2) : 0;
      }
      const int phys = p.paged ? __shfl_sync(0xffffffffu, pid_reg, k & 31) : 0;
      if (tile >= nts) continue;  // past the session's length (consumers skip it too)
      ++n;
      const int tile_end_key = tile * KT + KT;
      const unsigned need = __ballot_sync(0xffffffffu, lane < sg.n_ag && tile_end_key > my_a);
      const unsigned umask = p.mode == LRKV_BASE_SHARED ? need : (need ? 1u : 0u);
      const bool page_ok = !p.paged || (phys >= 0 && phys < p.num_pages);
      const uint32_t bytes = (page_ok ? 2 * KV_BYTES : 0) + __popc(umask) * U_BYTES;
      const bool freed = mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.flags, p.spin_cap, true);
      // After an abort the consumers release stages without waiting for their
      // copies, so nothing more may be issued: a stage could receive a second
      // copy while the first is still landing.  The abort word is read after the
      // wait (whose acquire orders it), and the whole warp leaves together.
      if (__any_sync(0xffffffffu, !freed || *abort_flag)) {
        stop = true;
        --n;  // this tile was not issued
        break;
      }
      if (lane == 0) {
        if (!page_ok) atomicOr(p.flags, LRKV_DEVFLAG_PAGE);
        seq[stage] = n - 1;
        uint8_t* st = ring + (size_t)stage * stage_bytes;
        if (bytes == 0) {
          mbar_arrive(&full[stage]);
        } else {
          mbar_arrive_expect_tx(&full[stage], bytes);
          if (page_ok) {
            const int c1 = p.paged ? 0 : tile * KT;
            const int c3 = p.paged ? phys : sg.s;
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
              tma_load_4d(st + hh * (KT * 128), tmK, &full[stage], hh * 64, c1, sg.g, c3, pol_kv);
              tma_load_4d(st + KV_BYTES + hh * (KT * 128), tmV, &full[stage], hh * 64, c1, sg.g, c3, pol_kv);
            }
          }
          unsigned m = umask;
          while (m) {
            const int slot = __ffs(m) - 1;
            m &= m - 1;
            const int agent_slot = p.mode == LRKV_BASE_SHARED ? sg.i_lo + slot : 0;
            tma_load_4d(st + 2 * KV_BYTES + slot * U_BYTES, tmU, &full[stage], 0, tile * KT, agent_slot, sg.s,
                        pol_u);
          }
        }
      }
      __syncwarp();
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  // After an abort the consumers may stop waiting; make sure no copy issued by
  // this CTA is still landing in shared memory when the CTA exits.
  if (*abort_flag && lane == 0) {
    const int m = n < p.stages ? n : p.stages;
    int st = stage;
    uint32_t ph = phase;
    for (int j = 0; j < m; ++j) {
      if (--st < 0) {
        st = p.stages - 1;
        ph ^= 1;
      }
      uint32_t spins = 0;
      while (!mbar_try_wait(&full[st], ph) && ++spins < kSpinCap) {
      }
    }
  }
}

// ---------------------------------------------------------------------------
// consumer warps
// ---------------------------------------------------------------------------
// NOG groups of NT warps.  Tile n of the CTA belongs to group n % NOG; warp
// w of a group owns query rows [8 w, 8 w + 8) of the work item and runs them
// over all 64 keys of its group's tiles.  The groups hold the same rows for
// different tiles and are merged at the end of a segment.
template <int D, int RK>
struct RowState {
  static constexpr int MT = D / 16;
  static constexpr int MTZ = RK >= 16 ? RK / 16 : 1;
  float m[2];
  // row sums as the accumulator of (all-ones 16 x 16) x P^T: l[0], l[1] are rows
  // 2 t4 and 2 t4 + 1, complete over every key of the segment; l[2], l[3] repeat them
  float l[4];       // rows 2 t4, 2 t4 + 1 of the warp's 8
  float o[MT][4];         // O^T: dims (16 mt + g8, + 8) x rows
  float z[MTZ][4];        // Z^T: ranks x rows
};

// Record layout: [m(RP) | l(RP) | O(RP x D) | Z(RP x RK)], rows r0.. of this warp.
template <int D, int RK>
__device__ __forceinline__ void store_rows(const RowState<D, RK>& st, float* rec, int RP, int rbase, int g8, int t4) {
  float* mO = rec + 2 * RP;
  float* mZ = mO + RP * D;
  const int r0 = rbase + 2 * t4;
  if (g8 == 0) {
    rec[r0] = st.m[0];
    rec[r0 + 1] = st.m[1];
    rec[RP + r0] = st.l[0];
    rec[RP + r0 + 1] = st.l[1];
  }
#pragma unroll
  for (int mt = 0; mt < RowState<D, RK>::MT; ++mt) {
    const int d0 = mt * 16 + g8;
    mO[r0 * D + d0] = st.o[mt][0];
    mO[(r0 + 1) * D + d0] = st.o[mt][1];
    mO[r0 * D + d0 + 8] = st.o[mt][2];
    mO[(r0 + 1) * D + d0 + 8] = st.o[mt][3];
  }
#pragma unroll
  for (int mz = 0; mz < RowState<D, RK>::MTZ; ++mz) {
    const int k0 = mz * 16 + g8;
    mZ[r0 * RK + k0] = st.z[mz][0];
    mZ[(r0 + 1) * RK + k0] = st.z[mz][1];
    if (k0 + 8 < RK) {
      mZ[r0 * RK + k0 + 8] = st.z[mz][2];
      mZ[(r0 + 1) * RK + k0 + 8] = st.z[mz][3];
    }
  }
}

// st <- the online-softmax combination of st and the stored rows.
template <int D, int RK>
__device__ __forceinline__ void absorb_rows(RowState<D, RK>& st, const float* rec, int RP, int rbase, int g8, int t4) {
  const float* mO = rec + 2 * RP;
  const float* mZ = mO + RP * D;
  const float NEG_INF = -INFINITY;
  const int r0 = rbase + 2 * t4;
  float sa[2], so[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float mo = rec[r0 + e];
    const float M = fmaxf(st.m[e], mo);
    sa[e] = st.m[e] == NEG_INF ? 0.f : fast_exp2(st.m[e] - M);
    so[e] = mo == NEG_INF ? 0.f : fast_exp2(mo - M);
    st.l[e] = st.l[e] * sa[e] + rec[RP + r0 + e] * so[e];
    st.m[e] = M;
  }
#pragma unroll
  for (int mt = 0; mt < RowState<D, RK>::MT; ++mt) {
    const int d0 = mt * 16 + g8;
    st.o[mt][0] = st.o[mt][0] * sa[0] + mO[r0 * D + d0] * so[0];
    st.o[mt][1] = st.o[mt][1] * sa[1] + mO[(r0 + 1) * D + d0] * so[1];
    st.o[mt][2] = st.o[mt][2] * sa[0] + mO[r0 * D + d0 + 8] * so[0];
    st.o[mt][3] = st.o[mt][3] * sa[1] + mO[(r0 + 1) * D + d0 + 8] * so[1];
  }
#pragma unroll
  for (int mz = 0; mz < RowState<D, RK>::MTZ; ++mz) {
    const int k0 = mz * 16 + g8;
    st.z[mz][0] = st.z[mz][0] * sa[0] + mZ[r0 * RK + k0] * so[0];
    st.z[mz][1] = st.z[mz][1] * sa[1] + mZ[(r0 + 1) * RK + k0] * so[1];
    if (k0 + 8 < RK) {
      st.z[mz][2] = st.z[mz][2] * sa[0] + mZ[r0 * RK + k0 + 8] * so[0];
      st.z[mz][3] = st.z[mz][3] * sa[1] + mZ[(r0 + 1) * RK + k0 + 8] * so[1];
    }
  }
}

// This warp's query rows as the B operand of S^T = K Q^T: row `qrow` of the
// item, dims 16 ks + 2 t4 (+1, +8, +9).
template <int D>
__device__ __forceinline__ void load_q_frags(const DecodeParams& p, const Seg& sg, int qrow, int t4,
                                             uint32_t (*qf)[2]) {
  const bool qvalid = qrow < sg.rows;
  const __nv_bfloat16* qptr = nullptr;
  if (qvalid) {
    const int grow = sg.row_lo + qrow;
    qptr = static_cast<const __nv_bfloat16*>(p.q) + (((size_t)sg.s * p.N + grow / p.G) * p.Hq + (p.g_base + sg.g) * p.G + grow % p.G) * D;
  }
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qf[ks][0] = qvalid ? __ldg(reinterpret_cast<const unsigned int*>(qptr + ks * 16 + 2 * t4)) : 0u;
    qf[ks][1] = qvalid ? __ldg(reinterpret_cast<const unsigned int*>(qptr + ks * 16 + 8 + 2 * t4)) : 0u;
  }
}

// Facts of one segment's merged record, enough to publish or finish it.
struct SegInfo {
  int item, s, g, row_lo, rows, i_lo, n_ag;
  int segs;  // CTAs sharing the item
  int slot;  // this CTA's partial-record slot among them
};

__device__ __forceinline__ SegInfo seg_info(const DecodeParams& p, const Seg& sg) {
  SegInfo si;
  si.item = sg.item;
  si.s = sg.s;
  si.g = sg.g;
  si.row_lo = sg.row_lo;
  si.rows = sg.rows;
  si.i_lo = sg.i_lo;
  si.n_ag = sg.n_ag;
  const long long C = gridDim.x;
  const long long c_first = owner_cta((long long)sg.item * p.nt, p.W, C);
  const long long c_last = owner_cta((long long)(sg.item + 1) * p.nt - 1, p.W, C);
  si.segs = (int)(c_last - c_first + 1);
  si.slot = (int)((long long)blockIdx.x - c_first);
  return si;
}

// Publish a segment's merged record `rec` (shared memory, [m | l | O | Z] per
// row), or, when this CTA is the last of the item's CTAs to get there (atomic
// ticket), combine every partial record of the item and write
// out = (O + Z B_i,g) / l: the up-projection of Eq. 12, once per row.  Run by a
// team of NTH threads (tid in [0, NTH)) that `sync` synchronises.
template <int D, int NT, int RK, int NTH, typename Sync>
__device__ __forceinline__ void finish_segment(const DecodeParams& p, const SegInfo& si, float* rec, float* scw,
                                               int* bcast, int tid, Sync sync) {
  constexpr int RP = NT * 8;
  constexpr int REC = RP * (D + RK + 2);
  constexpr int E4 = RP * (D + RK) / 4;
  constexpr int PERC = 6;  // float4 elements per thread per combine pass
  constexpr int D2 = D / 2;
  const float NEG_INF = -INFINITY;
  const int HD = p.Hkv_total * D;  // B rows span every KV head
  const int n_units = si.n_ag * D2;  // (agent, pair of adjacent dims)
  // B columns of the (agent, dim pair) units this thread will write
  auto b_col = [&](int u) {
    return reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.b) +
                                             ((size_t)(si.i_lo + u / D2) * RK) * HD + (size_t)(p.g_base + si.g) * D +
                                             2 * (u % D2));
  };
  // Bring this thread's first unit's B columns into L1 now (no registers held),
  // so that their latency overlaps the publish, the ticket and the combine.
  if (tid < n_units) {
    const uint32_t* bp = b_col(tid);
#pragma unroll
    for (int r = 0; r < RK; ++r) asm volatile("prefetch.L1 [%0];" ::"l"(bp + (size_t)r * (HD / 2)));
  }
  bool finish = true;
  if (si.segs > 1) {
    float* grec = p.partials + ((size_t)si.item * p.max_segs + (size_t)si.slot) * REC;
    for (int e = tid * 4; e < REC; e += NTH * 4)
      __stcg(reinterpret_cast<float4*>(grec + e), *reinterpret_cast<const float4*>(rec + e));
    sync();
    if (tid == 0) {
      __threadfence();
      const int prev = atomicAdd(p.tickets + si.item, 1);
      const int last = prev == si.segs - 1;
      if (last) p.tickets[si.item] = 0;
      *bcast = last;
    }
    sync();
    finish = *bcast != 0;
    if (!finish) return;
    __threadfence();
    const float* base = p.partials + (size_t)si.item * p.max_segs * REC;
    // With at most SEG_CHUNK records, one round of loads gives every record's
    // maximum and sum, hence the scales and l, before the O and Z pass; more
    // records take a pass for the maxima and then a scale table per chunk.
    const bool one_chunk = si.segs <= SEG_CHUNK;
    if (one_chunk) {
      if (tid < RP) {
        float mj[SEG_CHUNK], lj[SEG_CHUNK];
#pragma unroll
        for (int jj = 0; jj < SEG_CHUNK; ++jj) {
          mj[jj] = jj < si.segs ? __ldcg(base + (size_t)jj * REC + tid) : NEG_INF;
          lj[jj] = jj < si.segs ? __ldcg(base + (size_t)jj * REC + RP + tid) : 0.f;
        }
        float M = NEG_INF;
#pragma unroll
        for (int jj = 0; jj < SEG_CHUNK; ++jj) M = fmaxf(M, mj[jj]);
        float L = 0.f;
#pragma unroll
        for (int jj = 0; jj < SEG_CHUNK; ++jj) {
          const float sc = mj[jj] == NEG_INF ? 0.f : fast_exp2(mj[jj] - M);
          scw[jj * RP + tid] = sc;
          L += lj[jj] * sc;
        }
        rec[RP + tid] = L;
      }
    } else if (tid < RP) {  // maxima of every record, chunk by chunk; rows <= 32 <= NTH
      float M = NEG_INF;
      for (int j0 = 0; j0 < si.segs; j0 += SEG_CHUNK) {
        float mj[SEG_CHUNK];
#pragma unroll
        for (int jj = 0; jj < SEG_CHUNK; ++jj)
          mj[jj] = j0 + jj < si.segs ? __ldcg(base + (size_t)(j0 + jj) * REC + tid) : NEG_INF;
#pragma unroll
        for (int jj = 0; jj < SEG_CHUNK; ++jj) M = fmaxf(M, mj[jj]);
      }
      rec[tid] = M;
    }
    sync();
    // O and Z: PERC float4 per thread per pass, all records' loads of a pass issued together
    for (int e0 = 0; e0 < E4; e0 += NTH * PERC) {
      float4 acc[PERC];
#pragma unroll
      for (int u = 0; u < PERC; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      float L = 0.f;
      for (int j0 = 0; j0 < si.segs; j0 += SEG_CHUNK) {
        const int nj = min(SEG_CHUNK, si.segs - j0);
        if (!one_chunk) {
          if (tid < RP) {
            const float M = rec[tid];
#pragma unroll
            for (int jj = 0; jj < SEG_CHUNK; ++jj) {
              const float mj = jj < nj ? __ldcg(base + (size_t)(j0 + jj) * REC + tid) : NEG_INF;
              const float lj = jj < nj ? __ldcg(base + (size_t)(j0 + jj) * REC + RP + tid) : 0.f;
              const float sc = mj == NEG_INF ? 0.f : fast_exp2(mj - M);
              scw[jj * RP + tid] = sc;
              L += lj * sc;
            }
          }
          sync();
        }
        // records in groups of RG, the loads of a group issued together (one
        // round trip to L2 per group instead of one per record); the sums run
        // in record order either way
        constexpr int RG = NT >= 4 ? 2 : 4;  // the 32-row instance has the fewest registers to spare
        for (int jg = 0; jg < nj; jg += RG) {
          float4 v[RG][PERC];
#pragma unroll
          for (int q = 0; q < RG; ++q) {
            const float4* rj = reinterpret_cast<const float4*>(base + (size_t)(j0 + jg + q) * REC + 2 * RP);
#pragma unroll
            for (int u = 0; u < PERC; ++u) {
              const int e4 = e0 + tid + u * NTH;
              v[q][u] = (jg + q < nj && e4 < E4) ? __ldcg(rj + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
#pragma unroll
          for (int q = 0; q < RG; ++q) {
            if (jg + q >= nj) break;
#pragma unroll
            for (int u = 0; u < PERC; ++u) {
              const int e4 = e0 + tid + u * NTH;
              if (e4 >= E4) continue;
              const int e = e4 * 4;
              const int row = e < RP * D ? e / D : (e - RP * D) / RK;
              const float sc = scw[(jg + q) * RP + row];
              acc[u].x += v[q][u].x * sc;
              acc[u].y += v[q][u].y * sc;
              acc[u].z += v[q][u].z * sc;
              acc[u].w += v[q][u].w * sc;
            }
          }
        }
        if (!one_chunk) sync();  // the next chunk rewrites the scale table
      }
#pragma unroll
      for (int u = 0; u < PERC; ++u) {
        const int e4 = e0 + tid + u * NTH;
        if (e4 < E4) *reinterpret_cast<float4*>(rec + 2 * RP + e4 * 4) = acc[u];
      }
      if (!one_chunk && e0 == 0 && tid < RP) rec[RP + tid] = L;
    }
    sync();
  }
  // out = (O + Z B_i,g) / l.  A thread takes (agent, two adjacent dims): the
  // agent's B columns (bf16 pairs) serve all its GQA rows, a Z row is read as
  // float4s (the same row across the warp), O and the output go as pairs.
  const float* mL = rec + RP;
  const float* mO = rec + 2 * RP;
  const float* mZ = mO + RP * D;
  if (tid < RP) scw[tid] = mL[tid] > 0.f ? 1.f / mL[tid] : 0.f;  // 1 / l per row (the scale table is free)
  sync();
  const int h0 = (p.g_base + si.g) * p.G;
  for (int u = tid; u < n_units; u += NTH) {
    const int agent = si.i_lo + u / D2;
    const int dim = 2 * (u % D2);
    const uint32_t* bp = b_col(u);
    float b0[RK], b1[RK];
#pragma unroll
    for (int r = 0; r < RK; ++r) {
      const uint32_t w = __ldg(bp + (size_t)r * (HD / 2));
      b0[r] = __uint_as_float(w << 16);
      b1[r] = __uint_as_float(w & 0xffff0000u);
    }
    int r_begin = agent * p.G - si.row_lo, r_end = r_begin + p.G;
    r_begin = r_begin < 0 ? 0 : r_begin;
    r_end = r_end > si.rows ? si.rows : r_end;
    for (int row = r_begin; row < r_end; ++row) {
      float2 o = *reinterpret_cast<const float2*>(mO + row * D + dim);
      const float4* z4 = reinterpret_cast<const float4*>(mZ + row * RK);
#pragma unroll
      for (int q = 0; q < RK / 4; ++q) {
        const float4 z = z4[q];
        o.x = fmaf(z.x, b0[4 * q], o.x);
        o.y = fmaf(z.x, b1[4 * q], o.y);
        o.x = fmaf(z.y, b0[4 * q + 1], o.x);
        o.y = fmaf(z.y, b1[4 * q + 1], o.y);
        o.x = fmaf(z.z, b0[4 * q + 2], o.x);
        o.y = fmaf(z.z, b1[4 * q + 2], o.y);
        o.x = fmaf(z.w, b0[4 * q + 3], o.x);
        o.y = fmaf(z.w, b1[4 * q + 3], o.y);
      }
      const float il = scw[row];
      o.x *= il;
      o.y *= il;
      const int grow = si.row_lo + row;
      const size_t oi = (((size_t)si.s * p.N + agent) * p.Hq + h0 + grow % p.G) * D + dim;
      if (p.out_f32) *reinterpret_cast<float2*>(static_cast<float*>(p.out) + oi) = o;
      else *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.out) + oi) = __floats2bfloat162_rn(o.x, o.y);
    }
  }
}

template <int D, int NT, int RK, int NOG>
__device__ void decode_consumers(const DecodeParams& p, uint8_t* smem, const DecodeSmem& lay, uint64_t* full,
                                 uint64_t* empty, volatile int* seq, volatile int* abort_flag, int* bcast,
                                 long long t_begin, long long t_end) {
  constexpr int RP = NT * 8;
  constexpr int KS = D / 16;
  constexpr int MT = D / 16;
  constexpr int MTZ = RK >= 16 ? RK / 16 : 1;
  constexpr int KV_BYTES = KT * D * 2;
  constexpr int U_BYTES = KT * RK * 2;
  constexpr int REC = RP * (D + RK + 2);
  constexpr int CT = NOG * NT * 32;   // consumer threads
  const int tid = threadIdx.x;        // consumers are warps 0 .. NOG*NT-1
  const int warp = tid >> 5, lane = tid & 31;
  const int og = warp / NT;           // owner group
  const int nw = warp % NT;           // n-tile (8 rows) of this warp
  const int rbase = nw * 8;
  const int g8 = lane >> 2, t4 = lane & 3;
  const uint32_t ring_s = smem_u32(smem);
  int* a_sm = reinterpret_cast<int*>(smem + lay.a_off);
  const float NEG_INF = -INFINITY;

  int stage = 0;
  uint32_t phase = 0;
  int ntile = 0;  // tiles seen by this CTA so far (all groups)
  int sn = 0;     // segments of this CTA so far

  // Per-lane byte offsets of the ldmatrix rows inside a 128B-swizzled K/V
  // tile (64 keys x 64 dims per half): 16-byte chunk c of key row k sits at
  // chunk c ^ (k & 7).  koff[i] serves k-steps with (2 ks) & 7 == 2 i (K
  // operand), voff[i] serves m-tiles with (2 mt) & 7 == 2 i (V^T operand);
  // the key block (2048 B) and the 64-dim half (8192 B) are added as constants.
  uint32_t koff[4], voff[4];
  {
    const int j = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      koff[i] = ((j & 1) * 8 + r8) * 128 + ((((2 * i) + (j >> 1)) ^ r8) << 4);
      voff[i] = ((j >> 1) * 8 + r8) * 128 + ((((2 * i) + (j & 1)) ^ r8) << 4);
    }
  }

  uint32_t qf[KS][2];
  for (long long t = t_begin; t < t_end;) {
    Seg sg = make_seg(p, t, t_end, tid == 0);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    const int nts = seg_tiles_valid(sg);
    const int sl = sg.sl;

    if (tid < sg.n_ag) a_sm[tid] = load_offset(p, sg.s, sg.i_lo + tid, true);
    // this warp's query rows as the B operand of S^T = K Q^T (kept in registers;
    // from the second segment on they were fetched during the previous merge)
    const int qrow = rbase + g8;  // row of this lane's B fragment
    const bool qvalid = qrow < sg.rows;
    if (sn == 0) load_q_frags<D>(p, sg, qrow, t4, qf);
    named_bar_sync(1, CT);
    int a_max = 0;
    for (int j = 0; j < sg.n_ag; ++j) a_max = max(a_max, a_sm[j]);
    // agents whose rows meet this warp's 8 rows, and this lane's row's agent
    const int w_row_lo = sg.row_lo + rbase;
    const int w_rows = min(8, sg.rows - rbase);
    const int ag_lo = w_rows > 0 ? w_row_lo / p.G - sg.i_lo : 0;
    const int ag_hi = w_rows > 0 ? (w_row_lo + w_rows - 1) / p.G - sg.i_lo : -1;
    const int my_agent = qvalid ? (sg.row_lo + qrow) / p.G - sg.i_lo : -1;
    // the first key any of this warp's agents keeps a U row for: tiles wholly
    // before it skip the low-rank passes at one compare
    int a_first = 0x7fffffff;
    for (int ag = ag_lo; ag <= ag_hi; ++ag) a_first = min(a_first, a_sm[ag]);

    RowState<D, RK> st;
    st.m[0] = st.m[1] = NEG_INF;
    st.l[0] = st.l[1] = st.l[2] = st.l[3] = 0.f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[mt][e] = 0.f;
#pragma unroll
    for (int mz = 0; mz < MTZ; ++mz)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.z[mz][e] = 0.f;

    TileOrder ord = tile_order(p, sg.lo);
    for (int kk = sg.lo; kk < sg.hi; ++kk, ord.next()) {
      const int tile = ord.tile();
      if (tile >= nts) continue;  // past the session's length (the producer skips it too)
      const int my_n = ntile;
      const bool mine = (ntile % NOG) == og;
      const int my_stage = stage;
      const uint32_t my_phase = phase;
      ++ntile;
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
      if (!mine) continue;
      // wait until the producer has issued this tile into the stage, then for its bytes
      {
        uint32_t spins = 0;
        while (seq[my_stage] != my_n) {
          if (*abort_flag || ++spins >= p.spin_cap) {
            if (!*abort_flag) {
              *abort_flag = 1;
              atomicOr(p.flags, LRKV_DEVFLAG_TIMEOUT);
            }
            break;
          }
        }
      }
      mbar_wait_bounded(&full[my_stage], my_phase, abort_flag, p.flags, p.spin_cap, true);  // most tiles have landed
      const uint32_t Ks = ring_s + my_stage * lay.stage_bytes;
      const uint32_t Vs = Ks + KV_BYTES;
      const uint32_t Us = Vs + KV_BYTES;
      const int tile_key0 = tile * KT;

      // ---- S^T = K Q^T : 4 blocks of 16 keys x this warp's 8 rows (4 independent chains)
      float sacc[4][4];
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[kb][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t kb_base = Ks + koff[ks & 3] + (ks >> 2) * (KT * 128);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a0, a1, a2, a3, kb_base + kb * (16 * 128));
          mma_bf16_16816(sacc[kb], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        }
      }

      // ---- online softmax over the 64 keys (rows are columns of S^T).
      // The reference max of a row only moves when the tile max exceeds it by
      // more than 2^8 (log2 units): probabilities then stay <= 2^8 and the
      // accumulators need rescaling only on those rare tiles.  The result is
      // exact either way, since numerator and denominator share the reference.
      const bool boundary = tile_key0 + KT > sl;
      float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        if (boundary) {  // keys at or past seq_len are selected out
          const bool va = tile_key0 + 16 * kb + g8 < sl;
          const bool vb = tile_key0 + 16 * kb + g8 + 8 < sl;
          sacc[kb][0] = va ? sacc[kb][0] : NEG_INF;
          sacc[kb][1] = va ? sacc[kb][1] : NEG_INF;
          sacc[kb][2] = vb ? sacc[kb][2] : NEG_INF;
          sacc[kb][3] = vb ? sacc[kb][3] : NEG_INF;
        }
        mx0 = fmaxf(mx0, fmaxf(sacc[kb][0], sacc[kb][2]));
        mx1 = fmaxf(mx1, fmaxf(sacc[kb][1], sacc[kb][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      // the scale is positive and rounding monotonic: the max of the scaled
      // scores is the scaled max, and each weight takes the scale in one fma
      mx0 *= p.scale_log2;
      mx1 *= p.scale_log2;
      const bool need = (mx0 > st.m[0] + 8.f) || (mx1 > st.m[1] + 8.f);
      if (__any_sync(0xffffffffu, need)) {
        float al[2];
        const float mxv[2] = {mx0, mx1};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float mn = fmaxf(st.m[e], mxv[e]);
          al[e] = mn == NEG_INF ? 1.f : fast_exp2(st.m[e] - mn);
          st.m[e] = mn;
          st.l[e] *= al[e];
          st.l[e + 2] *= al[e];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          st.o[mt][0] *= al[0];
          st.o[mt][1] *= al[1];
          st.o[mt][2] *= al[0];
          st.o[mt][3] *= al[1];
        }
#pragma unroll
        for (int mz = 0; mz < MTZ; ++mz) {
          st.z[mz][0] *= al[0];
          st.z[mz][1] *= al[1];
          st.z[mz][2] *= al[0];
          st.z[mz][3] *= al[1];
        }
      }
      const float mu0 = st.m[0] == NEG_INF ? 0.f : st.m[0];
      const float mu1 = st.m[1] == NEG_INF ? 0.f : st.m[1];
      uint32_t pb[4][2];
      const float sc = p.scale_log2;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        const float p0 = fast_exp2(fmaf(sacc[kb][0], sc, -mu0)), p1 = fast_exp2(fmaf(sacc[kb][1], sc, -mu1));
        const float p2 = fast_exp2(fmaf(sacc[kb][2], sc, -mu0)), p3 = fast_exp2(fmaf(sacc[kb][3], sc, -mu1));
        pb[kb][0] = movmatrix_t(pack_bf16x2(p0, p1));
        pb[kb][1] = movmatrix_t(pack_bf16x2(p2, p3));
        // the row sums of exactly the bf16 weights the value MMA uses: ones x P^T
        constexpr uint32_t kOnes = 0x3F803F80u;  // two bf16 1.0
        mma_bf16_16816(st.l, kOnes, kOnes, kOnes, kOnes, pb[kb][0], pb[kb][1]);
      }

      // ---- O^T += V^T P^T ; V rows past seq_len are selected out
      uint32_t vm[4][2];
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        vm[kb][0] = vm[kb][1] = 0xffffffffu;
        if (boundary) {
          const int k0 = tile_key0 + 16 * kb + 2 * t4;
          vm[kb][0] = (k0 < sl ? 0x0000ffffu : 0u) | (k0 + 1 < sl ? 0xffff0000u : 0u);
          vm[kb][1] = (k0 + 8 < sl ? 0x0000ffffu : 0u) | (k0 + 9 < sl ? 0xffff0000u : 0u);
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const uint32_t mt_base = Vs + voff[mt & 3] + (mt >> 2) * (KT * 128);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(a0, a1, a2, a3, mt_base + kb * (16 * 128));
          if (boundary) {
            a0 &= vm[kb][0];
            a1 &= vm[kb][0];
            a2 &= vm[kb][1];
            a3 &= vm[kb][1];
          }
          mma_bf16_16816(st.o[mt], a0, a1, a2, a3, pb[kb][0], pb[kb][1]);
        }
      }

      // ---- Z^T += U_i^T P^T over this warp's rows of agent i; U rows < a_i or >= seq_len selected out.
      // Tiles wholly inside [a_i, seq_len) need no masks: one ldmatrix and one MMA per key block.
      const bool lr_full = p.mode == LRKV_BASE_LR_SHARED && !boundary && a_max <= tile_key0;
      const int pass_lo = lr_full ? 0 : ag_lo;
      const int pass_hi = lr_full ? 0 : (tile_key0 + KT > a_first ? ag_hi : ag_lo - 1);
      for (int ag = pass_lo; ag <= pass_hi; ++ag) {
        const int a_i = lr_full ? 0 : a_sm[ag];
        if (tile_key0 + KT <= a_i) continue;  // producer did not load this U tile
        const int slot = p.mode == LRKV_BASE_SHARED ? ag : 0;
        const uint32_t ub = Us + slot * U_BYTES;
        const bool use = lr_full ? (my_agent >= 0) : (my_agent == ag);
        const bool clean = !boundary && a_i <= tile_key0;  // warp-uniform
        uint32_t bz[4][2];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          bz[kb][0] = use ? pb[kb][0] : 0u;
          bz[kb][1] = use ? pb[kb][1] : 0u;
        }
        if (clean) {
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
            for (int mz = 0; mz < MTZ; ++mz) {
              uint32_t a0, a1 = 0, a2, a3 = 0;
              if constexpr (RK == 8) {
                ldsm_x2_t(a0, a2, ub + (16 * kb + ((lane >> 3) & 1) * 8 + (lane & 7)) * (RK * 2));
              } else {
                const int j = lane >> 3;
                ldsm_x4_t(a0, a1, a2, a3,
                          ub + (16 * kb + (j >> 1) * 8 + (lane & 7)) * (RK * 2) + (2 * mz + (j & 1)) * 16);
              }
              mma_bf16_16816(st.z[mz], a0, a1, a2, a3, bz[kb][0], bz[kb][1]);
            }
          }
          continue;
        }
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          const int k16 = tile_key0 + 16 * kb;
          if (k16 + 16 <= a_i || k16 >= sl) continue;  // warp-uniform
          const int k0 = k16 + 2 * t4;
          const bool ok0 = k0 >= a_i && k0 < sl, ok1 = k0 + 1 >= a_i && k0 + 1 < sl;
          const bool ok8 = k0 + 8 >= a_i && k0 + 8 < sl, ok9 = k0 + 9 >= a_i && k0 + 9 < sl;
          const uint32_t um_lo = (ok0 ? 0x0000ffffu : 0u) | (ok1 ? 0xffff0000u : 0u);
          const uint32_t um_hi = (ok8 ? 0x0000ffffu : 0u) | (ok9 ? 0xffff0000u : 0u);
#pragma unroll
          for (int mz = 0; mz < MTZ; ++mz) {
            uint32_t a0, a1 = 0, a2, a3 = 0;
            if constexpr (RK == 8) {
              ldsm_x2_t(a0, a2, ub + (16 * kb + ((lane >> 3) & 1) * 8 + (lane & 7)) * (RK * 2));
            } else {
              const int j = lane >> 3;
              ldsm_x4_t(a0, a1, a2, a3,
                        ub + (16 * kb + (j >> 1) * 8 + (lane & 7)) * (RK * 2) + (2 * mz + (j & 1)) * 16);
            }
            a0 &= um_lo;
            a1 &= um_lo;
            a2 &= um_hi;
            a3 &= um_hi;
            mma_bf16_16816(st.z[mz], a0, a1, a2, a3, bz[kb][0], bz[kb][1]);
          }
        }
      }

      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[my_stage]);
    }

    // ---- segment end.  The next segment's query fragments are fetched now so
    // that their latency overlaps the merge.  The addresses used here are
    // formed here rather than kept live through the tile loop, and the last
    // segment's B columns are loaded inside the finish rather than held in
    // registers across the merge: the tile loop needs every register.
    const bool last_seg = t >= t_end;
    const int buf = sn & 1;
    float* merge = reinterpret_cast<float*>(smem + lay.merge_off) + buf * REC;  // records alternate
    uint64_t* rec_full = full + 2 * p.stages;
    uint64_t* rec_free = rec_full + 2;
    if (!last_seg) {
      Seg nx = make_seg(p, t, t_end, false);
      seg_rows(p, nx);
      load_q_frags<D>(p, nx, rbase + g8, t4, qf);
    }
    // the record buffer of segment sn - 2 must have been released by the epilogue warp
    if (sn >= 2) mbar_wait_bounded(&rec_free[buf], ((sn >> 1) - 1) & 1, abort_flag, p.flags, p.spin_cap);
    // chain the owner groups into the record (same rows, different tiles)
    for (int src = NOG - 1; src >= 1; --src) {
      if (og == src) store_rows<D, RK>(st, merge, RP, rbase, g8, t4);
      named_bar_sync(1, CT);
      if (og == src - 1) absorb_rows<D, RK>(st, merge, RP, rbase, g8, t4);
      named_bar_sync(1, CT);
    }
    if (og == 0) store_rows<D, RK>(st, merge, RP, rbase, g8, t4);
    named_bar_sync(1, CT);
    if (!last_seg) {
      // hand the record to the epilogue warp and go on streaming
      if (tid == 0) mbar_arrive(&rec_full[buf]);
    } else {
      const SegInfo si = seg_info(p, sg);
      float* scw = reinterpret_cast<float*>(smem + lay.scw_off);  // the consumers' half
      finish_segment<D, NT, RK, CT>(p, si, merge, scw, bcast, tid, [] { named_bar_sync(1, CT); });
    }
    ++sn;
  }
}

// The epilogue warp: publishes (and, as the last CTA of an item, combines and
// finishes) the records of every segment of this CTA but the last, while the
// consumer warps stream the next segment's tiles.
template <int D, int NT, int RK>
__device__ void decode_epilogue(const DecodeParams& p, uint8_t* smem, const DecodeSmem& lay, uint64_t* rec_full,
                                uint64_t* rec_free, volatile int* abort_flag, int* bcast, long long t_begin,
                                long long t_end) {
  constexpr int RP = NT * 8;
  constexpr int REC = RP * (D + RK + 2);
  const int lane = threadIdx.x & 31;
  float* merge0 = reinterpret_cast<float*>(smem + lay.merge_off);
  float* scw = reinterpret_cast<float*>(smem + lay.scw_off) + 8 * RP;  // the epilogue warp's half
  int sn = 0;
  for (long long t = t_begin; t < t_end;) {
    Seg sg = make_seg(p, t, t_end, false);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    if (t >= t_end) break;  // the consumers finish the last segment
    const int buf = sn & 1;
    if (!mbar_wait_bounded(&rec_full[buf], (sn >> 1) & 1, abort_flag, p.flags, p.spin_cap)) break;
    const SegInfo si = seg_info(p, sg);
    finish_segment<D, NT, RK, 32>(p, si, merge0 + buf * REC, scw, bcast, lane, [] { __syncwarp(); });
    __syncwarp();
    if (lane == 0) mbar_arrive(&rec_free[buf]);
    ++sn;
  }
}

// Warp roles: warps 0 .. NOG*NT-1 consume (NOG owner groups of NT warps), then
// one producer warp and one epilogue warp.
template <int NT, int NOG>
struct Roles {
  static constexpr int CONSUMER_WARPS = NOG * NT;
  static constexpr int THREADS = (CONSUMER_WARPS + 2) * 32;
};

template <int D, int NT, int RK, int NOG>
__global__ void __launch_bounds__(Roles<NT, NOG>::THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmU, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const DecodeSmem lay = decode_smem_plan(D, NT, RK, p.n_u_slots, p.stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* rec_full = empty + p.stages;
  uint64_t* rec_free = rec_full + 2;
  volatile int* seq = reinterpret_cast<volatile int*>(rec_free + 2);
  volatile int* abort_flag = seq + p.stages;
  int* bcast = const_cast<int*>(abort_flag) + 1;  // [0] consumers, [1] epilogue warp
  const int warp = threadIdx.x >> 5;
  constexpr int PRODUCER = Roles<NT, NOG>::CONSUMER_WARPS;
  constexpr int EPILOGUE = PRODUCER + 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NT);  // the NT warps of the group that owns the tile
      seq[s] = -1;
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&rec_full[b], 1);
      mbar_init(&rec_free[b], 1);
    }
    *abort_flag = 0;
    bcast[0] = bcast[1] = 0;
    fence_barrier_init();
  }
  if (warp == PRODUCER && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmU);
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  const long long C = gridDim.x;
  const long long t_begin = (long long)blockIdx.x * p.W / C;
  const long long t_end = (long long)(blockIdx.x + 1) * p.W / C;
  if (warp == PRODUCER) {
    decode_producer<D, RK>(p, &tmK, &tmV, &tmU, smem, lay.stage_bytes, full, empty, seq, abort_flag, t_begin,
                           t_end);
  } else if (warp == EPILOGUE) {
    decode_epilogue<D, NT, RK>(p, smem, lay, rec_full, rec_free, abort_flag, bcast + 1, t_begin, t_end);
  } else {
    decode_consumers<D, NT, RK, NOG>(p, smem, lay, full, empty, seq, abort_flag, bcast, t_begin, t_end);
  }
}

template <int D, int NT, int RK, int NOG>
lrkv_status launch_one(const DecodeParams& p, const void* tmK, const void* tmV, const void* tmU, int smem,
                       int ctas, cudaStream_t stream) {
  auto kern = decode_kernel<D, NT, RK, NOG>;
  if (ensure_dynamic_smem<decode_kernel<D, NT, RK, NOG>>(smem) != cudaSuccess) return LRKV_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(Roles<NT, NOG>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap& k = *static_cast<const CUtensorMap*>(tmK);
  const CUtensorMap& v = *static_cast<const CUtensorMap*>(tmV);
  const CUtensorMap& u = *static_cast<const CUtensorMap*>(tmU);
  if (cudaLaunchKernelEx(&cfg, kern, k, v, u, p) != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

template <int D, int RK>
lrkv_status dispatch_nt(const DecodeParams& p, int NT, int groups, const void* tmK, const void* tmV, const void* tmU,
                        int smem, int ctas, cudaStream_t st) {
  if (groups != decode_groups(NT, false) && groups != decode_groups(NT, true)) return LRKV_ERR_UNSUPPORTED;
  switch (NT) {
    case 1:
      return groups == 4 ? launch_one<D, 1, RK, 4>(p, tmK, tmV, tmU, smem, ctas, st)
                         : launch_one<D, 1, RK, 3>(p, tmK, tmV, tmU, smem, ctas, st);
    case 2: return launch_one<D, 2, RK, 3>(p, tmK, tmV, tmU, smem, ctas, st);
    case 3: return launch_one<D, 3, RK, 2>(p, tmK, tmV, tmU, smem, ctas, st);
    case 4: return launch_one<D, 4, RK, 2>(p, tmK, tmV, tmU, smem, ctas, st);
  }
  return LRKV_ERR_UNSUPPORTED;
}

}  // namespace

lrkv_status launch_decode(const DecodeParams& p, int D, int NT, int RK, int groups, const void* tmK, const void* tmV,
                          const void* tmU, int smem_bytes, int ctas, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128) {
    if (RK == 8) return dispatch_nt<128, 8>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 16) return dispatch_nt<128, 16>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 32) return dispatch_nt<128, 32>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
  } else if (D == 64) {
    if (RK == 8) return dispatch_nt<64, 8>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 16) return dispatch_nt<64, 16>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 32) return dispatch_nt<64, 32>(p, NT, groups, tmK, tmV, tmU, smem_bytes, ctas, st);
  }
  return LRKV_ERR_UNSUPPORTED;
}

}  // namespace lrkv
