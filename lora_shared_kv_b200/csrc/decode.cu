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
constexpr int NCW = 4;                     // consumer warps
constexpr int DEC_THREADS = (NCW + 1) * 32;
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
template <int D, int NT, int RK>
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
  const int tid = threadIdx.x;  // 0..127
  const int warp = tid >> 5, lane = tid & 31;
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

  for (long long t = t_begin; t < t_end;) {
    Seg sg = make_seg(p, t, t_end, tid == 0);
    t += sg.hi - sg.lo;
    seg_rows(p, sg);
    const int hi_e = seg_tiles_end(sg);
    const int sl = sg.sl;

    // ---- stage this item's queries (rows x d, 16B chunks, XOR-swizzled) and offsets
    {
      constexpr int CH = D / 8;
      for (int idx = tid; idx < RP * CH; idx += NCW * 32) {
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
      named_bar_sync(1, NCW * 32);
    }
    int a_max = 0;
    for (int j = 0; j < sg.n_ag; ++j) a_max = max(a_max, a_sm[j]);
    int my_agent[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r = nt * 8 + g8;
      my_agent[nt] = r < sg.rows ? (sg.row_lo + r) / p.G - sg.i_lo : -1;
    }

    float m_run[NT][2], l_run[NT][2];
    float oacc[MT][NT][4];
    float zacc[MTZ][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_run[nt][0] = m_run[nt][1] = NEG_INF;
      l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][nt][e] = 0.f;
#pragma unroll
      for (int mz = 0; mz < MTZ; ++mz)
#pragma unroll
        for (int e = 0; e < 4; ++e) zacc[mz][nt][e] = 0.f;
    }

    for (int tile = sg.lo; tile < hi_e; ++tile) {
      mbar_wait_bounded(&full[stage], phase, abort_flag, p.flags);
      const uint32_t Ks = ring_s + stage * lay.stage_bytes;
      const uint32_t Vs = Ks + KV_BYTES;
      const uint32_t Us = Vs + KV_BYTES;
      const int kbase = tile * KT + 16 * warp;

      // ---- S^T = K Q^T : 16 keys x RP rows per warp
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ks += 2) {
        uint32_t a[2][4];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int j = lane >> 3;
          const int key = 16 * warp + (j & 1) * 8 + (lane & 7);
          const int ch = (ks + kk) * 2 + (j >> 1);
          const uint32_t addr = Ks + (ch >> 3) * (KT * 128) + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
          ldsm_x4(a[kk][0], a[kk][1], a[kk][2], a[kk][3], addr);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int row = nt * 8 + (lane & 7);
          const int ch = ks * 2 + (lane >> 3);
          const uint32_t addr = q_s + row * (D * 2) + (((ch & ~7) | ((ch & 7) ^ (row & 7))) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3, addr);
          mma_bf16_16816(sacc[nt], a[0][0], a[0][1], a[0][2], a[0][3], b0, b1);
          mma_bf16_16816(sacc[nt], a[1][0], a[1][1], a[1][2], a[1][3], b2, b3);
        }
      }

      // ---- online softmax over this warp's 16 keys (rows are columns of S^T)
      const int key_a = kbase + g8, key_b = key_a + 8;
      const bool va = key_a < sl, vb = key_b < sl;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float s0 = va ? sacc[nt][0] * p.scale_log2 : NEG_INF;
        float s1 = va ? sacc[nt][1] * p.scale_log2 : NEG_INF;
        float s2 = vb ? sacc[nt][2] * p.scale_log2 : NEG_INF;
        float s3 = vb ? sacc[nt][3] * p.scale_log2 : NEG_INF;
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
        const float mu0 = mn0 == NEG_INF ? 0.f : mn0, mu1 = mn1 == NEG_INF ? 0.f : mn1;
        const float al0 = fast_exp2(m_run[nt][0] - mu0), al1 = fast_exp2(m_run[nt][1] - mu1);
        m_run[nt][0] = mn0;
        m_run[nt][1] = mn1;
        const float p0 = fast_exp2(s0 - mu0), p1 = fast_exp2(s1 - mu1);
        const float p2 = fast_exp2(s2 - mu0), p3 = fast_exp2(s3 - mu1);
        l_run[nt][0] = l_run[nt][0] * al0 + (p0 + p2);
        l_run[nt][1] = l_run[nt][1] * al1 + (p1 + p3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          oacc[mt][nt][0] *= al0;
          oacc[mt][nt][1] *= al1;
          oacc[mt][nt][2] *= al0;
          oacc[mt][nt][3] *= al1;
        }
#pragma unroll
        for (int mz = 0; mz < MTZ; ++mz) {
          zacc[mz][nt][0] *= al0;
          zacc[mz][nt][1] *= al1;
          zacc[mz][nt][2] *= al0;
          zacc[mz][nt][3] *= al1;
        }
        pb[nt][0] = movmatrix_t(pack_bf16x2(p0, p1));
        pb[nt][1] = movmatrix_t(pack_bf16x2(p2, p3));
      }

      // ---- O^T += V^T P^T ; V rows past seq_len are selected out
      const bool boundary = tile * KT + KT > sl;
      uint32_t vm_lo = 0xffffffffu, vm_hi = 0xffffffffu;
      if (boundary) {
        const int k0 = kbase + 2 * t4;
        vm_lo = (k0 < sl ? 0x0000ffffu : 0u) | (k0 + 1 < sl ? 0xffff0000u : 0u);
        vm_hi = (k0 + 8 < sl ? 0x0000ffffu : 0u) | (k0 + 9 < sl ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int j = lane >> 3;
        const int key = 16 * warp + (j >> 1) * 8 + (lane & 7);
        const int ch = 2 * mt + (j & 1);
        const uint32_t addr = Vs + (ch >> 3) * (KT * 128) + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(a0, a1, a2, a3, addr);
        a0 &= vm_lo;
        a1 &= vm_lo;
        a2 &= vm_hi;
        a3 &= vm_hi;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(oacc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }

      // ---- Z^T += U_i^T P^T over rows of agent i; U rows < a_i or >= seq_len selected out
      const int tile_key0 = tile * KT;
      if (tile_key0 + KT > 0) {
        const bool lr_full = p.mode == LRKV_BASE_LR_SHARED && !boundary && a_max <= tile_key0;
        for (int ag = 0; ag < (lr_full ? 1 : sg.n_ag); ++ag) {
          const int a_i = lr_full ? 0 : a_sm[ag];
          if (tile_key0 + KT <= a_i) continue;         // producer did not load this U tile
          if (kbase + 16 <= a_i || kbase >= sl) continue;  // nothing of this warp's slice is adapted
          const int slot = p.mode == LRKV_BASE_SHARED ? ag : 0;
          const uint32_t ub = Us + slot * U_BYTES;
          const int k0 = kbase + 2 * t4;
          const bool ok0 = k0 >= a_i && k0 < sl, ok1 = k0 + 1 >= a_i && k0 + 1 < sl;
          const bool ok8 = k0 + 8 >= a_i && k0 + 8 < sl, ok9 = k0 + 9 >= a_i && k0 + 9 < sl;
          const uint32_t um_lo = (ok0 ? 0x0000ffffu : 0u) | (ok1 ? 0xffff0000u : 0u);
          const uint32_t um_hi = (ok8 ? 0x0000ffffu : 0u) | (ok9 ? 0xffff0000u : 0u);
#pragma unroll
          for (int mz = 0; mz < MTZ; ++mz) {
            uint32_t a0, a1 = 0, a2, a3 = 0;
            if constexpr (RK == 8) {
              const int key = 16 * warp + ((lane >> 3) & 1) * 8 + (lane & 7);
              ldsm_x2_t(a0, a2, ub + key * (RK * 2));
            } else {
              const int j = lane >> 3;
              const int key = 16 * warp + (j >> 1) * 8 + (lane & 7);
              const int ch = 2 * mz + (j & 1);
              ldsm_x4_t(a0, a1, a2, a3, ub + key * (RK * 2) + ch * 16);
            }
            a0 &= um_lo;
            a1 &= um_lo;
            a2 &= um_hi;
            a3 &= um_hi;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const bool mine = lr_full ? (my_agent[nt] >= 0) : (my_agent[nt] == ag);
              const uint32_t b0 = mine ? pb[nt][0] : 0u, b1 = mine ? pb[nt][1] : 0u;
              // skip n-tiles holding none of this agent's rows (warp-uniform test)
              if (!lr_full) {
                const int r_first = (sg.i_lo + ag) * p.G - sg.row_lo;
                const int r_last = r_first + p.G - 1;
                if (r_last < nt * 8 || r_first > nt * 8 + 7) continue;
              }
              mma_bf16_16816(zacc[mz][nt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }

      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
    }

    // ---- per-warp state -> shared memory (rows x [m, l, O, Z])
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l_run[nt][e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        l_run[nt][e] = v;
      }
    {
      float* mr = merge + warp * REC;
      float* mO = mr + 2 * RP;
      float* mZ = mO + RP * D;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int r0 = nt * 8 + 2 * t4;
        if (g8 == 0) {
          mr[r0] = m_run[nt][0];
          mr[r0 + 1] = m_run[nt][1];
          mr[RP + r0] = l_run[nt][0];
          mr[RP + r0 + 1] = l_run[nt][1];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int d0 = mt * 16 + g8;
          mO[r0 * D + d0] = oacc[mt][nt][0];
          mO[(r0 + 1) * D + d0] = oacc[mt][nt][1];
          mO[r0 * D + d0 + 8] = oacc[mt][nt][2];
          mO[(r0 + 1) * D + d0 + 8] = oacc[mt][nt][3];
        }
#pragma unroll
        for (int mz = 0; mz < MTZ; ++mz) {
          const int k0 = mz * 16 + g8;
          mZ[r0 * RK + k0] = zacc[mz][nt][0];
          mZ[(r0 + 1) * RK + k0] = zacc[mz][nt][1];
          if (k0 + 8 < RK) {
            mZ[r0 * RK + k0 + 8] = zacc[mz][nt][2];
            mZ[(r0 + 1) * RK + k0 + 8] = zacc[mz][nt][3];
          }
        }
      }
    }
    named_bar_sync(1, NCW * 32);

    // ---- merge the four warps into record 0
    if (tid < RP) {
      float M = NEG_INF;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, merge[w * REC + tid]);
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = merge[w * REC + tid];
        const float sc = mw == NEG_INF ? 0.f : fast_exp2(mw - M);
        scw[w * RP + tid] = sc;
        L += merge[w * REC + RP + tid] * sc;
      }
      merge[tid] = M;
      merge[RP + tid] = L;
    }
    named_bar_sync(1, NCW * 32);
    for (int e = tid; e < RP * (D + RK); e += NCW * 32) {
      const int row = e < RP * D ? e / D : (e - RP * D) / RK;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) v += merge[w * REC + 2 * RP + e] * scw[w * RP + row];
      merge[2 * RP + e] = v;
    }
    named_bar_sync(1, NCW * 32);

    // ---- publish or finish this item
    const long long W = p.W;
    const long long c_first = owner_cta((long long)sg.item * p.nt, W, C);
    const long long c_last = owner_cta((long long)(sg.item + 1) * p.nt - 1, W, C);
    const int segs = (int)(c_last - c_first + 1);
    bool finish = true;
    if (segs > 1) {
      float* rec = p.partials + ((size_t)sg.item * p.max_segs + (size_t)(c - c_first)) * REC;
      for (int e = tid * 4; e < REC; e += NCW * 32 * 4)
        __stcg(reinterpret_cast<float4*>(rec + e), *reinterpret_cast<const float4*>(merge + e));
      named_bar_sync(1, NCW * 32);
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(p.tickets + sg.item, 1);
        const int last = prev == segs - 1;
        if (last) p.tickets[sg.item] = 0;
        *bcast = last;
      }
      named_bar_sync(1, NCW * 32);
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
        named_bar_sync(1, NCW * 32);
        for (int j0 = 0; j0 < segs; j0 += SEG_CHUNK) {
          const int nj = min(SEG_CHUNK, segs - j0);
          if (tid < RP) {
            const float M = merge[tid];
            for (int jj = 0; jj < nj; ++jj) {
              const float mj = __ldcg(base + (size_t)(j0 + jj) * REC + tid);
              scw[jj * RP + tid] = mj == NEG_INF ? 0.f : fast_exp2(mj - M);
            }
          }
          named_bar_sync(1, NCW * 32);
          for (int e = tid; e < RP * (D + RK); e += NCW * 32) {
            const int row = e < RP * D ? e / D : (e - RP * D) / RK;
            float v = j0 == 0 ? 0.f : merge[2 * RP + e];
            for (int jj = 0; jj < nj; ++jj) v += __ldcg(base + (size_t)(j0 + jj) * REC + 2 * RP + e) * scw[jj * RP + row];
            merge[2 * RP + e] = v;
          }
          named_bar_sync(1, NCW * 32);
        }
      }
    }

    if (finish) {
      // out = (O + Z B_i,g) / l, once per row: the up-projection of Eq. 12
      const float* mL = merge + RP;
      const float* mO = merge + 2 * RP;
      const float* mZ = mO + RP * D;
      const int HD = p.Hkv * D;
      for (int e = tid; e < sg.rows * D; e += NCW * 32) {
        const int row = e / D, dim = e % D;
        const int grow = sg.row_lo + row;
        const int agent = grow / p.G;
        const int h = sg.g * p.G + grow % p.G;
        const uint16_t* bcol =
            static_cast<const uint16_t*>(p.b) + ((size_t)agent * RK) * HD + (size_t)sg.g * D + dim;
        float acc = mO[row * D + dim];
#pragma unroll
        for (int k = 0; k < RK; ++k) acc = fmaf(mZ[row * RK + k], bf16_to_f32(__ldg(bcol + (size_t)k * HD)), acc);
        const float L = mL[row];
        const float o = L > 0.f ? acc / L : 0.f;
        const size_t oi = (((size_t)sg.s * p.N + agent) * p.Hq + h) * D + dim;
        if (p.out_f32) static_cast<float*>(p.out)[oi] = o;
        else static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
      }
    }
    named_bar_sync(1, NCW * 32);
  }
}

template <int D, int NT, int RK>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmU, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const DecodeSmem lay = decode_smem_plan(D, NT, RK, p.n_u_slots, p.stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar_off);
  uint64_t* empty = full + p.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + p.stages);
  int* bcast = const_cast<int*>(abort_flag) + 1;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    *bcast = 0;
    fence_barrier_init();
  }
  if (warp == NCW && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmU);
  }
  __syncthreads();
  pdl_wait();
  const long long C = gridDim.x;
  const long long t_begin = (long long)blockIdx.x * p.W / C;
  const long long t_end = (long long)(blockIdx.x + 1) * p.W / C;
  if (warp == NCW) {
    decode_producer<D, RK>(p, &tmK, &tmV, &tmU, smem, lay.stage_bytes, full, empty, abort_flag, t_begin, t_end);
  } else {
    decode_consumers<D, NT, RK>(p, smem, lay, full, empty, abort_flag, bcast, t_begin, t_end);
  }
  pdl_launch_dependents();
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
  cfg.blockDim = dim3(DEC_THREADS);
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

int decode_threads() { return DEC_THREADS; }

}  // namespace lrkv
