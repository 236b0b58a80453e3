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
//    to finish it (atomic ticket), which also applies Z B_i and the 1/l.
//  * A producer warp moves 64-key K/V tiles (128B-swizzled) and the rank-r U
//    tiles with the Tensor Memory Accelerator into a ring of stages guarded by
//    mbarriers.  U tiles wholly before an agent's offset are never loaded.
//  * Four consumer warps each own 16 keys of every tile and run the
//    contractions on the tensor cores with keys as the M dimension
//    (S^T = K Q^T, O^T += V^T P^T, Z^T += U_i^T P^T), so a handful of query
//    rows pads only to a multiple of 8.  The score accumulators are
//    re-laid into the P^T operand with movmatrix; the online-softmax row
//    reductions are warp shuffles.  Rows past seq_len and U rows before a_i
//    are removed by selects on the operands, never by multiplying with 0.
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

__device__ __forceinline__ int seg_tiles_end(const Seg& sg) {
  const int nts = (sg.sl + KT - 1) / KT;
  return sg.hi < nts ? sg.hi : nts;
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
template <int D, int RK>
__device__ void decode_producer(const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                const CUtensorMap* tmU, uint8_t* ring, int stage_bytes, uint64_t* full,
                                uint64_t* empty, volatile int* abort_flag, long long t_begin, long long t_end) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = policy_evict_first();
  const uint64_t pol_u = policy_evict_last();
  constexpr int KV_BYTES = KT * D * 2;
  constexpr int U_BYTES = KT * RK * 2;
  int stage = 0;
  uint32_t phase = 0;
  long long issued = 0;
  for (long long t = t_begin; t < t_end;) {
    Seg sg = make_seg(p, t, t_end, false);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    const int hi_e = seg_tiles_end(sg);
    // lane j < n_ag holds the offset of agent i_lo + j
    const int my_a = lane < sg.n_ag ? load_offset(p, sg.s, sg.i_lo + lane, false) : 0x7fffffff;
    int pid_reg = 0;
    for (int tile = sg.lo; tile < hi_e; ++tile) {
      const int k = tile - sg.lo;
      if (p.paged && (k & 31) == 0) {
        const int tt = tile + lane;
        pid_reg = tt < hi_e ? __ldg(p.page_table + (size_t)sg.s * p.pt_stride + tt) : 0;
      }
      const int phys = p.paged ? __shfl_sync(0xffffffffu, pid_reg, k & 31) : 0;
      const int tile_end_key = tile * KT + KT;
      const unsigned need = __ballot_sync(0xffffffffu, lane < sg.n_ag && tile_end_key > my_a);
      unsigned umask;
      if (p.mode == LRKV_BASE_SHARED) umask = need;
      else umask = need ? 1u : 0u;
      const bool page_ok = !p.paged || (phys >= 0 && phys < p.num_pages);
      const uint32_t bytes = (page_ok ? 2 * KV_BYTES : 0) + __popc(umask) * U_BYTES;
      mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.flags);
      if (lane == 0) {
        if (!page_ok) atomicOr(p.flags, LRKV_DEVFLAG_PAGE);
        uint8_t* st = ring + (size_t)stage * stage_bytes;
        if (bytes == 0) {
          mbar_arrive(&full[stage]);
        } else {
          mbar_arrive_expect_tx(&full[stage], bytes);
          if (page_ok) {
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
              const int c1 = p.paged ? 0 : tile * KT;
              const int c3 = p.paged ? phys : sg.s;
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
      ++issued;
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  // After an abort the consumers may stop waiting; make sure no copy issued by
  // this CTA is still landing in shared memory when the CTA exits.
  if (*abort_flag && lane == 0) {
    long long n = issued < p.stages ? issued : p.stages;
    int st = stage;
    uint32_t ph = phase;
    for (long long j = 0; j < n; ++j) {
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
// NG warpgroups of four warps.  Tile n of the CTA (counted over all its
// segments) belongs to group n % NG; warp w of a group owns keys
// [16 w, 16 w + 16) of its tiles.  Each warp keeps its own online-softmax
// state; the states are merged in shared memory at the end of a segment.
template <int D, int NT, int RK>
struct WarpState {
  static constexpr int MT = D / 16;
  static constexpr int MTZ = RK >= 16 ? RK / 16 : 1;
  float m[NT][2], l[NT][2];
  float o[MT][NT][4];
  float z[MTZ][NT][4];
};

// Write a warp's state (l already reduced over its lanes) to a record
// [m(RP) | l(RP) | O(RP x D) | Z(RP x RK)].
template <int D, int NT, int RK>
__device__ __forceinline__ void store_state(const WarpState<D, NT, RK>& st, float* mr, int g8, int t4) {
  constexpr int RP = NT * 8;
  float* mO = mr + 2 * RP;
  float* mZ = mO + RP * D;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int r0 = nt * 8 + 2 * t4;
    if (g8 == 0) {
      mr[r0] = st.m[nt][0];
      mr[r0 + 1] = st.m[nt][1];
      mr[RP + r0] = st.l[nt][0];
      mr[RP + r0 + 1] = st.l[nt][1];
    }
#pragma unroll
    for (int mt = 0; mt < WarpState<D, NT, RK>::MT; ++mt) {
      const int d0 = mt * 16 + g8;
      mO[r0 * D + d0] = st.o[mt][nt][0];
      mO[(r0 + 1) * D + d0] = st.o[mt][nt][1];
      mO[r0 * D + d0 + 8] = st.o[mt][nt][2];
      mO[(r0 + 1) * D + d0 + 8] = st.o[mt][nt][3];
    }
#pragma unroll
    for (int mz = 0; mz < WarpState<D, NT, RK>::MTZ; ++mz) {
      const int k0 = mz * 16 + g8;
      mZ[r0 * RK + k0] = st.z[mz][nt][0];
      mZ[(r0 + 1) * RK + k0] = st.z[mz][nt][1];
      if (k0 + 8 < RK) {
        mZ[r0 * RK + k0 + 8] = st.z[mz][nt][2];
        mZ[(r0 + 1) * RK + k0 + 8] = st.z[mz][nt][3];
      }
    }
  }
}

// st <- merge(st, record): the online-softmax combination of two partial states.
template <int D, int NT, int RK>
__device__ __forceinline__ void absorb_state(WarpState<D, NT, RK>& st, const float* mr, int g8, int t4) {
  constexpr int RP = NT * 8;
  const float* mO = mr + 2 * RP;
  const float* mZ = mO + RP * D;
  const float NEG_INF = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int r0 = nt * 8 + 2 * t4;
    float sa[2], so[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float mo = mr[r0 + e];
      const float M = fmaxf(st.m[nt][e], mo);
      sa[e] = st.m[nt][e] == NEG_INF ? 0.f : fast_exp2(st.m[nt][e] - M);
      so[e] = mo == NEG_INF ? 0.f : fast_exp2(mo - M);
      st.l[nt][e] = st.l[nt][e] * sa[e] + mr[RP + r0 + e] * so[e];
      st.m[nt][e] = M;
    }
#pragma unroll
    for (int mt = 0; mt < WarpState<D, NT, RK>::MT; ++mt) {
      const int d0 = mt * 16 + g8;
      st.o[mt][nt][0] = st.o[mt][nt][0] * sa[0] + mO[r0 * D + d0] * so[0];
      st.o[mt][nt][1] = st.o[mt][nt][1] * sa[1] + mO[(r0 + 1) * D + d0] * so[1];
      st.o[mt][nt][2] = st.o[mt][nt][2] * sa[0] + mO[r0 * D + d0 + 8] * so[0];
      st.o[mt][nt][3] = st.o[mt][nt][3] * sa[1] + mO[(r0 + 1) * D + d0 + 8] * so[1];
    }
#pragma unroll
    for (int mz = 0; mz < WarpState<D, NT, RK>::MTZ; ++mz) {
      const int k0 = mz * 16 + g8;
      st.z[mz][nt][0] = st.z[mz][nt][0] * sa[0] + mZ[r0 * RK + k0] * so[0];
      st.z[mz][nt][1] = st.z[mz][nt][1] * sa[1] + mZ[(r0 + 1) * RK + k0] * so[1];
      if (k0 + 8 < RK) {
        st.z[mz][nt][2] = st.z[mz][nt][2] * sa[0] + mZ[r0 * RK + k0 + 8] * so[0];
        st.z[mz][nt][3] = st.z[mz][nt][3] * sa[1] + mZ[(r0 + 1) * RK + k0 + 8] * so[1];
      }
    }
  }
}

template <int D, int NT, int RK, int NG>
__device__ void decode_consumers(const DecodeParams& p, uint8_t* smem, const DecodeSmem& lay, uint64_t* full,
                                 uint64_t* empty, volatile int* abort_flag, int* bcast, long long t_begin,
                                 long long t_end) {
  constexpr int RP = NT * 8;
  constexpr int KS = D / 16;
  constexpr int MT = D / 16;
  constexpr int MTZ = RK >= 16 ? RK / 16 : 1;
  constexpr int KV_BYTES = KT * D * 2;
  constexpr int U_BYTES = KT * RK * 2;
  constexpr int REC = RP * (D + RK + 2);
  constexpr int CT = NG * 4 * 32;  // consumer threads
  const int tid = threadIdx.x - 128;  // 0 .. CT-1 (warpgroup 0 is the producer)
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int NOG = NG * 2;      // owner groups: pairs of warps, tile n goes to pair n % NOG
  static_assert(NOG == (NT <= 3 ? 2 : 1) * 2, "owner groups must match decode_owner_groups()");
  const int og = warp >> 1;        // owner group of this warp
  const int kh = warp & 1;         // key half (32 of the 64 keys of a tile) of this warp
  const int g8 = lane >> 2, t4 = lane & 3;
  const uint32_t ring_s = smem_u32(smem);
  const uint32_t q_s = smem_u32(smem + lay.q_off);
  float* merge = reinterpret_cast<float*>(smem + lay.merge_off);
  float* scw = reinterpret_cast<float*>(smem + lay.scw_off);
  int* a_sm = reinterpret_cast<int*>(smem + lay.a_off);
  const float NEG_INF = -INFINITY;
  const long long C = gridDim.x;
  const long long c = blockIdx.x;

  int stage = 0;
  uint32_t phase = 0;
  int ntile = 0;  // tiles seen by this CTA so far (all groups)

  for (long long t = t_begin; t < t_end;) {
    Seg sg = make_seg(p, t, t_end, tid == 0);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    const int hi_e = seg_tiles_end(sg);
    const int sl = sg.sl;

    // ---- stage this item's queries (rows x d, 16B chunks, XOR-swizzled) and offsets
    {
      constexpr int CH = D / 8;
      for (int idx = tid; idx < RP * CH; idx += CT) {
        const int row = idx / CH, ch = idx % CH;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (row < sg.rows) {
          const int grow = sg.row_lo + row;
          const int agent = grow / p.G;
          const int h = sg.g * p.G + grow % p.G;
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) +
                                                            (((size_t)sg.s * p.N + agent) * p.Hq + h) * D) + ch;
          val = __ldg(src);
        }
        const int pch = (ch & ~7) | ((ch & 7) ^ (row & 7));
        *reinterpret_cast<uint4*>(smem + lay.q_off + row * (D * 2) + pch * 16) = val;
      }
      if (tid < sg.n_ag) a_sm[tid] = load_offset(p, sg.s, sg.i_lo + tid, true);
      named_bar_sync(1, CT);
    }
    int a_max = 0;
    for (int j = 0; j < sg.n_ag; ++j) a_max = max(a_max, a_sm[j]);
    int my_agent[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r = nt * 8 + g8;
      my_agent[nt] = r < sg.rows ? (sg.row_lo + r) / p.G - sg.i_lo : -1;
    }

    WarpState<D, NT, RK> st;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      st.m[nt][0] = st.m[nt][1] = NEG_INF;
      st.l[nt][0] = st.l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[mt][nt][e] = 0.f;
#pragma unroll
      for (int mz = 0; mz < MTZ; ++mz)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.z[mz][nt][e] = 0.f;
    }

    for (int tile = sg.lo; tile < hi_e; ++tile) {
      const bool mine = (ntile % NOG) == og;
      const int my_stage = stage;
      const uint32_t my_phase = phase;
      ++ntile;
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
      if (!mine) continue;
      mbar_wait_bounded(&full[my_stage], my_phase, abort_flag, p.flags);
      const uint32_t Ks = ring_s + my_stage * lay.stage_bytes;
      const uint32_t Vs = Ks + KV_BYTES;
      const uint32_t Us = Vs + KV_BYTES;
      const int kw = 32 * kh;                 // first key of this warp inside the tile
      const int kbase = tile * KT + kw;       // absolute key

      // ---- S^T = K Q^T : two 16-key blocks x RP rows (2 x NT independent chains)
      float sacc[2][NT][4];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[kb][nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ks += 2) {
        uint32_t a[2][2][4];  // [kb][k-step][reg]
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const int j = lane >> 3;
            const int key = kw + 16 * kb + (j & 1) * 8 + (lane & 7);
            const int ch = (ks + kk) * 2 + (j >> 1);
            const uint32_t addr = Ks + (ch >> 3) * (KT * 128) + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
            ldsm_x4(a[kb][kk][0], a[kb][kk][1], a[kb][kk][2], a[kb][kk][3], addr);
          }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int row = nt * 8 + (lane & 7);
          const int ch = ks * 2 + (lane >> 3);
          const uint32_t addr = q_s + row * (D * 2) + (((ch & ~7) | ((ch & 7) ^ (row & 7))) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3, addr);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            mma_bf16_16816(sacc[kb][nt], a[kb][0][0], a[kb][0][1], a[kb][0][2], a[kb][0][3], b0, b1);
            mma_bf16_16816(sacc[kb][nt], a[kb][1][0], a[kb][1][1], a[kb][1][2], a[kb][1][3], b2, b3);
          }
        }
      }

      // ---- online softmax over this warp's 32 keys (rows are columns of S^T).
      // The reference max of a row only moves when the tile max exceeds it by
      // more than 2^8 (log2 units): probabilities then stay <= 2^8 and the
      // accumulators need rescaling only on those rare tiles.  The result is
      // exact either way, since numerator and denominator share the reference.
      bool valid[2][2];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        valid[kb][0] = kbase + 16 * kb + g8 < sl;
        valid[kb][1] = kbase + 16 * kb + g8 + 8 < sl;
      }
      float mx[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          sacc[kb][nt][0] = valid[kb][0] ? sacc[kb][nt][0] * p.scale_log2 : NEG_INF;
          sacc[kb][nt][1] = valid[kb][0] ? sacc[kb][nt][1] * p.scale_log2 : NEG_INF;
          sacc[kb][nt][2] = valid[kb][1] ? sacc[kb][nt][2] * p.scale_log2 : NEG_INF;
          sacc[kb][nt][3] = valid[kb][1] ? sacc[kb][nt][3] * p.scale_log2 : NEG_INF;
        }
        mx[nt][0] = fmaxf(fmaxf(sacc[0][nt][0], sacc[0][nt][2]), fmaxf(sacc[1][nt][0], sacc[1][nt][2]));
        mx[nt][1] = fmaxf(fmaxf(sacc[0][nt][1], sacc[0][nt][3]), fmaxf(sacc[1][nt][1], sacc[1][nt][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mx[nt][0] = fmaxf(mx[nt][0], __shfl_xor_sync(0xffffffffu, mx[nt][0], o));
          mx[nt][1] = fmaxf(mx[nt][1], __shfl_xor_sync(0xffffffffu, mx[nt][1], o));
        }
      bool need = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        need |= (mx[nt][0] > st.m[nt][0] + 8.f) || (mx[nt][1] > st.m[nt][1] + 8.f);
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float al[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float mn = fmaxf(st.m[nt][e], mx[nt][e]);
            al[e] = mn == NEG_INF ? 1.f : fast_exp2(st.m[nt][e] - mn);
            st.m[nt][e] = mn;
            st.l[nt][e] *= al[e];
          }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            st.o[mt][nt][0] *= al[0];
            st.o[mt][nt][1] *= al[1];
            st.o[mt][nt][2] *= al[0];
            st.o[mt][nt][3] *= al[1];
          }
#pragma unroll
          for (int mz = 0; mz < MTZ; ++mz) {
            st.z[mz][nt][0] *= al[0];
            st.z[mz][nt][1] *= al[1];
            st.z[mz][nt][2] *= al[0];
            st.z[mz][nt][3] *= al[1];
          }
        }
      }
      uint32_t pb[2][NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float mu0 = st.m[nt][0] == NEG_INF ? 0.f : st.m[nt][0];
        const float mu1 = st.m[nt][1] == NEG_INF ? 0.f : st.m[nt][1];
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const float p0 = fast_exp2(sacc[kb][nt][0] - mu0), p1 = fast_exp2(sacc[kb][nt][1] - mu1);
          const float p2 = fast_exp2(sacc[kb][nt][2] - mu0), p3 = fast_exp2(sacc[kb][nt][3] - mu1);
          st.l[nt][0] += p0 + p2;
          st.l[nt][1] += p1 + p3;
          pb[kb][nt][0] = movmatrix_t(pack_bf16x2(p0, p1));
          pb[kb][nt][1] = movmatrix_t(pack_bf16x2(p2, p3));
        }
      }

      // ---- O^T += V^T P^T ; V rows past seq_len are selected out
      const bool boundary = tile * KT + KT > sl;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        uint32_t vm_lo = 0xffffffffu, vm_hi = 0xffffffffu;
        if (boundary) {
          const int k0 = kbase + 16 * kb + 2 * t4;
          vm_lo = (k0 < sl ? 0x0000ffffu : 0u) | (k0 + 1 < sl ? 0xffff0000u : 0u);
          vm_hi = (k0 + 8 < sl ? 0x0000ffffu : 0u) | (k0 + 9 < sl ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int j = lane >> 3;
          const int key = kw + 16 * kb + (j >> 1) * 8 + (lane & 7);
          const int ch = 2 * mt + (j & 1);
          const uint32_t addr = Vs + (ch >> 3) * (KT * 128) + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(a0, a1, a2, a3, addr);
          a0 &= vm_lo;
          a1 &= vm_lo;
          a2 &= vm_hi;
          a3 &= vm_hi;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16_16816(st.o[mt][nt], a0, a1, a2, a3, pb[kb][nt][0], pb[kb][nt][1]);
        }
      }

      // ---- Z^T += U_i^T P^T over rows of agent i; U rows < a_i or >= seq_len selected out
      const int tile_key0 = tile * KT;
      const bool lr_full = p.mode == LRKV_BASE_LR_SHARED && !boundary && a_max <= tile_key0;
      const int n_pass = lr_full ? 1 : sg.n_ag;
      for (int ag = 0; ag < n_pass; ++ag) {
        const int a_i = lr_full ? 0 : a_sm[ag];
        if (tile_key0 + KT <= a_i) continue;            // producer did not load this U tile
        if (kbase + 32 <= a_i || kbase >= sl) continue;  // nothing of this warp's keys is adapted
        const int slot = p.mode == LRKV_BASE_SHARED ? ag : 0;
        const uint32_t ub = Us + slot * U_BYTES;
        int nt_lo = 0, nt_hi = NT - 1;
        if (!lr_full) {
          const int r_first = (sg.i_lo + ag) * p.G - sg.row_lo;
          const int r_last = r_first + p.G - 1;
          nt_lo = r_first > 0 ? r_first / 8 : 0;
          nt_hi = r_last / 8 < NT - 1 ? r_last / 8 : NT - 1;
        }
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const int k16 = kbase + 16 * kb;
          if (k16 + 16 <= a_i || k16 >= sl) continue;
          const int k0 = k16 + 2 * t4;
          const bool ok0 = k0 >= a_i && k0 < sl, ok1 = k0 + 1 >= a_i && k0 + 1 < sl;
          const bool ok8 = k0 + 8 >= a_i && k0 + 8 < sl, ok9 = k0 + 9 >= a_i && k0 + 9 < sl;
          const uint32_t um_lo = (ok0 ? 0x0000ffffu : 0u) | (ok1 ? 0xffff0000u : 0u);
          const uint32_t um_hi = (ok8 ? 0x0000ffffu : 0u) | (ok9 ? 0xffff0000u : 0u);
#pragma unroll
          for (int mz = 0; mz < MTZ; ++mz) {
            uint32_t a0, a1 = 0, a2, a3 = 0;
            if constexpr (RK == 8) {
              const int key = kw + 16 * kb + ((lane >> 3) & 1) * 8 + (lane & 7);
              ldsm_x2_t(a0, a2, ub + key * (RK * 2));
            } else {
              const int j = lane >> 3;
              const int key = kw + 16 * kb + (j >> 1) * 8 + (lane & 7);
              const int ch = 2 * mz + (j & 1);
              ldsm_x4_t(a0, a1, a2, a3, ub + key * (RK * 2) + ch * 16);
            }
            a0 &= um_lo;
            a1 &= um_lo;
            a2 &= um_hi;
            a3 &= um_hi;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (nt < nt_lo || nt > nt_hi) continue;  // no row of this agent in this n-tile
              const bool use = lr_full ? (my_agent[nt] >= 0) : (my_agent[nt] == ag);
              const uint32_t b0 = use ? pb[kb][nt][0] : 0u, b1 = use ? pb[kb][nt][1] : 0u;
              mma_bf16_16816(st.z[mz][nt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }

      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[my_stage]);
    }

    // ---- reduce l over the lanes that share a row, then merge the warps:
    // owner groups pairwise (same key half), then the two key halves.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = st.l[nt][e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        st.l[nt][e] = v;
      }
    // a chain NOG-1 -> ... -> 1 -> 0 through one shared record per key half
    for (int src = NOG - 1; src >= 1; --src) {
      if (og == src) store_state<D, NT, RK>(st, merge + kh * REC, g8, t4);
      named_bar_sync(1, CT);
      if (og == src - 1) absorb_state<D, NT, RK>(st, merge + kh * REC, g8, t4);
      named_bar_sync(1, CT);
    }
    if (og == 0) store_state<D, NT, RK>(st, merge + kh * REC, g8, t4);
    named_bar_sync(1, CT);

    // ---- merge the two key halves into record 0
    if (tid < RP) {
      const float m0 = merge[tid], m1 = merge[REC + tid];
      const float M = fmaxf(m0, m1);
      const float s0 = m0 == NEG_INF ? 0.f : fast_exp2(m0 - M);
      const float s1 = m1 == NEG_INF ? 0.f : fast_exp2(m1 - M);
      scw[tid] = s0;
      scw[RP + tid] = s1;
      merge[RP + tid] = merge[RP + tid] * s0 + merge[REC + RP + tid] * s1;
      merge[tid] = M;
    }
    named_bar_sync(1, CT);
    for (int e4 = tid; e4 < RP * (D + RK) / 4; e4 += CT) {
      const int e = e4 * 4;
      const int row = e < RP * D ? e / D : (e - RP * D) / RK;
      const float4 x0 = *reinterpret_cast<const float4*>(merge + 2 * RP + e);
      const float4 x1 = *reinterpret_cast<const float4*>(merge + REC + 2 * RP + e);
      const float s0 = scw[row], s1 = scw[RP + row];
      *reinterpret_cast<float4*>(merge + 2 * RP + e) =
          make_float4(x0.x * s0 + x1.x * s1, x0.y * s0 + x1.y * s1, x0.z * s0 + x1.z * s1, x0.w * s0 + x1.w * s1);
    }
    named_bar_sync(1, CT);

    // ---- publish or finish this item
    const long long W = p.W;
    const long long c_first = owner_cta((long long)sg.item * p.nt, W, C);
    const long long c_last = owner_cta((long long)(sg.item + 1) * p.nt - 1, W, C);
    const int segs = (int)(c_last - c_first + 1);
    bool finish = true;
    if (segs > 1) {
      float* rec = p.partials + ((size_t)sg.item * p.max_segs + (size_t)(c - c_first)) * REC;
      for (int e = tid * 4; e < REC; e += CT * 4)
        __stcg(reinterpret_cast<float4*>(rec + e), *reinterpret_cast<const float4*>(merge + e));
      named_bar_sync(1, CT);
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(p.tickets + sg.item, 1);
        const int last = prev == segs - 1;
        if (last) p.tickets[sg.item] = 0;
        *bcast = last;
      }
      named_bar_sync(1, CT);
      finish = *bcast != 0;
      if (finish) {
        __threadfence();
        const float* base = p.partials + (size_t)sg.item * p.max_segs * REC;
        if (tid < RP) {
          float M = NEG_INF;
          for (int j = 0; j < segs; ++j) M = fmaxf(M, __ldcg(base + (size_t)j * REC + tid));
          float L = 0.f;
          for (int j = 0; j < segs; ++j) {
            const float mj = __ldcg(base + (size_t)j * REC + tid);
            L += mj == NEG_INF ? 0.f : __ldcg(base + (size_t)j * REC + RP + tid) * fast_exp2(mj - M);
          }
          merge[tid] = M;
          merge[RP + tid] = L;
        }
        named_bar_sync(1, CT);
        for (int j0 = 0; j0 < segs; j0 += SEG_CHUNK) {
          const int nj = min(SEG_CHUNK, segs - j0);
          if (tid < RP) {
            const float M = merge[tid];
            for (int jj = 0; jj < nj; ++jj) {
              const float mj = __ldcg(base + (size_t)(j0 + jj) * REC + tid);
              scw[jj * RP + tid] = mj == NEG_INF ? 0.f : fast_exp2(mj - M);
            }
          }
          named_bar_sync(1, CT);
          constexpr int E4 = RP * (D + RK) / 4;
          for (int e4 = tid; e4 < E4; e4 += 2 * CT) {
            float4 acc[2];
            int rows2[2];
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
              const int e = (e4 + u2 * CT) * 4;
              rows2[u2] = e < RP * D ? e / D : (e - RP * D) / RK;
              acc[u2] = (j0 == 0 || e4 + u2 * CT >= E4) ? make_float4(0.f, 0.f, 0.f, 0.f)
                                                          : *reinterpret_cast<const float4*>(merge + 2 * RP + e);
            }
            for (int jj = 0; jj < nj; ++jj) {
              const float* rj = base + (size_t)(j0 + jj) * REC + 2 * RP;
#pragma unroll
              for (int u2 = 0; u2 < 2; ++u2) {
                if (e4 + u2 * CT >= E4) continue;
                const float4 x = __ldcg(reinterpret_cast<const float4*>(rj + (e4 + u2 * CT) * 4));
                const float sc = scw[jj * RP + rows2[u2]];
                acc[u2].x += x.x * sc;
                acc[u2].y += x.y * sc;
                acc[u2].z += x.z * sc;
                acc[u2].w += x.w * sc;
              }
            }
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2)
              if (e4 + u2 * CT < E4) *reinterpret_cast<float4*>(merge + 2 * RP + (e4 + u2 * CT) * 4) = acc[u2];
          }
          named_bar_sync(1, CT);
        }
      }
    }

    if (finish) {
      // out = (O + Z B_i,g) / l, once per row: the up-projection of Eq. 12.
      // One thread per (agent, dim): the agent's B column is loaded once and
      // reused by every GQA row of that agent.
      const float* mL = merge + RP;
      const float* mO = merge + 2 * RP;
      const float* mZ = mO + RP * D;
      const int HD = p.Hkv * D;
      for (int e = tid; e < sg.n_ag * D; e += CT) {
        const int a_loc = e / D, dim = e % D;
        const int agent = sg.i_lo + a_loc;
        const uint16_t* bcol = static_cast<const uint16_t*>(p.b) + ((size_t)agent * RK) * HD + (size_t)sg.g * D + dim;
        float bk[RK];
#pragma unroll
        for (int k = 0; k < RK; ++k) bk[k] = bf16_to_f32(__ldg(bcol + (size_t)k * HD));
        int r_begin = agent * p.G - sg.row_lo, r_end = r_begin + p.G;
        r_begin = r_begin < 0 ? 0 : r_begin;
        r_end = r_end > sg.rows ? sg.rows : r_end;
        for (int row = r_begin; row < r_end; ++row) {
          float acc = mO[row * D + dim];
#pragma unroll
          for (int k = 0; k < RK; ++k) acc = fmaf(mZ[row * RK + k], bk[k], acc);
          const float L = mL[row];
          const float o = L > 0.f ? acc / L : 0.f;
          const int grow = sg.row_lo + row;
          const int h = sg.g * p.G + grow % p.G;
          const size_t oi = (((size_t)sg.s * p.N + agent) * p.Hq + h) * D + dim;
          if (p.out_f32) static_cast<float*>(p.out)[oi] = o;
          else static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
        }
      }
    }
    named_bar_sync(1, CT);
  }
}

// Warp roles: warpgroup 0 is the producer (one warp issues the copies, its
// register budget is cut to kProducerRegs), warpgroups 1..NG consume.  The
// block is launched with THREADS x kLaunchRegs registers; the split
// kProducerRegs x 128 + kConsumerRegs x 128 x NG must not exceed that total.
template <int NT>
struct Groups {
  static constexpr int NG = NT <= 3 ? 2 : 1;  // 32 padded rows need the whole register file: one group
  static constexpr int THREADS = (NG + 1) * 128;
};
constexpr int kLaunchRegs = 168;     // 65536 / 384, rounded down to a multiple of 8
constexpr int kProducerRegs = 32;
constexpr int kConsumerRegs = 232;
static_assert(kProducerRegs * 128 + kConsumerRegs * 256 <= kLaunchRegs * 384, "register split exceeds the launch");

template <int D, int NT, int RK>
__global__ void __launch_bounds__(Groups<NT>::THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmU, const DecodeParams p) {
  constexpr int NG = Groups<NT>::NG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const DecodeSmem lay = decode_smem_plan(D, NT, RK, p.n_u_slots, p.stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  uint64_t* empty = full + p.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + p.stages);
  int* bcast = const_cast<int*>(abort_flag) + 1;
  const int warp = threadIdx.x >> 5;
  if (p.stages % decode_owner_groups(NT) != 0) {  // every stage must keep one owner group
    if (threadIdx.x == 0) atomicOr(p.flags, LRKV_DEVFLAG_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // the two warps of the pair that owns the tile
    }
    *abort_flag = 0;
    *bcast = 0;
    fence_barrier_init();
  }
  if (warp == 0 && (threadIdx.x & 31) == 0) {
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
  if (warp < 4) {
    if constexpr (NG == 2) setmaxnreg_dec<kProducerRegs>();
    if (warp == 0)
      decode_producer<D, RK>(p, &tmK, &tmV, &tmU, smem, lay.stage_bytes, full, empty, abort_flag, t_begin, t_end);
  } else {
    if constexpr (NG == 2) setmaxnreg_inc<kConsumerRegs>();
    decode_consumers<D, NT, RK, NG>(p, smem, lay, full, empty, abort_flag, bcast, t_begin, t_end);
  }
}

template <int D, int NT, int RK>
lrkv_status launch_one(const DecodeParams& p, const void* tmK, const void* tmV, const void* tmU, int smem,
                       int ctas, cudaStream_t stream) {
  auto kern = decode_kernel<D, NT, RK>;
  static int configured_smem = 0;
  if (configured_smem < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return LRKV_ERR_CUDA;
    configured_smem = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(Groups<NT>::THREADS);
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
lrkv_status dispatch_nt(const DecodeParams& p, int NT, const void* tmK, const void* tmV, const void* tmU,
                        int smem, int ctas, cudaStream_t st) {
  switch (NT) {
    case 1: return launch_one<D, 1, RK>(p, tmK, tmV, tmU, smem, ctas, st);
    case 2: return launch_one<D, 2, RK>(p, tmK, tmV, tmU, smem, ctas, st);
    case 3: return launch_one<D, 3, RK>(p, tmK, tmV, tmU, smem, ctas, st);
    case 4: return launch_one<D, 4, RK>(p, tmK, tmV, tmU, smem, ctas, st);
  }
  return LRKV_ERR_UNSUPPORTED;
}

}  // namespace

lrkv_status launch_decode(const DecodeParams& p, int D, int NT, int RK, const void* tmK, const void* tmV,
                          const void* tmU, int smem_bytes, int ctas, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128) {
    if (RK == 8) return dispatch_nt<128, 8>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 16) return dispatch_nt<128, 16>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 32) return dispatch_nt<128, 32>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
  } else if (D == 64) {
    if (RK == 8) return dispatch_nt<64, 8>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 16) return dispatch_nt<64, 16>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
    if (RK == 32) return dispatch_nt<64, 32>(p, NT, tmK, tmV, tmU, smem_bytes, ctas, st);
  }
  return LRKV_ERR_UNSUPPORTED;
}

}  // namespace lrkv
