// Prefill-chunk attention over the shared base cache with per-agent low-rank
// value caches, on the 5th-generation tensor cores (tcgen05, TMEM).
//
// For agent i, query head h (KV head g = h / G) and chunk row j at absolute
// position L0 + j:
//     o = ( P V_base,g + (P Umask_i) B_i,g ) / l,   P = exp(q K_base,g^T * scale - m),  keys t <= L0 + j
// Eq. 12 of "LRAgent: Efficient KV Cache Sharing for Multi-LoRA LLM Agents"
// (Pith review, "What carries the argument"): the rank-r values are
// accumulated next to O as Z = P Umask_i and B_i is applied once per row, at
// the end.  Umask_i drops U rows before the agent's aLoRA offset ("RoleKV",
// "What it does").
//
// A 128-row tile is one agent, one KV head, floor(128/G) chunk tokens x the G
// query heads that share the KV head, so every K/V block loaded serves all of
// them (when G does not divide 128, the last 128 mod G rows are unused).
// The (tile, 128-key block) pairs are split evenly over one persistent CTA per
// SM (stream-K): a CTA walks a contiguous range of them, tile after tile, and
// a tile cut by a range boundary is finished by the last of its CTAs to get
// there (atomic ticket), which merges the others' partial (m, l, O + Z B) rows.
// Roles:
//   warp 0        TMA producer: B_i,g of each tile segment (double buffer),
//                 then its 128-key blocks of K into a 3-stage ring (a stage
//                 frees as soon as its S is computed).
//   warp 2        TMA producer of the V and U blocks (2-stage ring).
//   warp 1        TMEM owner and MMA issuer (one thread): S_j = Q K_j^T with
//                 the Q tile read from TMEM, into a double-buffered S; then
//                 [O | Z | l] += P_j [V_j | U_j | 1] with P_j read from TMEM
//                 (it overwrites S_j).  V_j, U_j and a constant block whose
//                 column 0 is one lie side by side in shared memory as one
//                 operand, so a k-step is one MMA of N = d + r + 16 and the row
//                 sums l of exactly the bf16 weights come out with O.  U rows
//                 before the aLoRA offset are zero-filled (the U of blocks
//                 wholly before it is not loaded).  At the end of a segment it
//                 adds Z B_i,g to O with two more MMA pairs (Z split into bf16
//                 high and low parts in TMEM, B_i,g in shared memory), so the
//                 epilogue only divides by l.
//   warps 4..11   Q into TMEM (the next segment's as soon as the last S of
//                 the current one has been read), softmax and epilogue, in two
//                 warpgroups, one per half of the block's 128 keys; a thread
//                 owns one row (TMEM lane) of its half.  The two warps of a
//                 lane quarter agree on each row's reference max through
//                 shared memory.  The reference max moves only when
//                 a block exceeds it by 2^8, and only then are O, Z and l
//                 rescaled in TMEM (each half rescales its share of the
//                 columns).  The epilogue splits the output columns.
#include <float.h>
#include <math.h>

#include "common.cuh"
#include "prefill.h"

namespace lrkv {

namespace {

// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

constexpr int BM = 128;   // rows per tile (TMEM lanes)
constexpr int BN = 128;   // keys per block
constexpr int KST = 3;    // K ring: a stage is free once S = Q K^T has been computed
constexpr int VST = 2;    // V/U ring: a stage is free once the PV MMA is done
constexpr int THREADS = 384;      // K producer, MMA, V/U producer, idle, 2 softmax warpgroups
constexpr int SMX_THREADS = 256;  // the two softmax warpgroups (named barrier 1); the two warps of
                                  // one 32-row lane quarter pair up on named barriers 2..5
constexpr uint32_t TMEM_COLS = 512;

template <int D, int RK>
struct PrefillLayout {
  static constexpr int B_BYTES = RK * D * 2;
  static constexpr int K_BYTES = BN * D * 2;
  static constexpr int U_BYTES = BN * RK * 2;
  // V block (D / RK atoms), the U block, then a constant atom whose column 0
  // is 1, so that the row sums of P come out of the same MMA as O and Z
  static constexpr int V_STAGE = K_BYTES + 2 * U_BYTES;
  static constexpr int U_OFF = K_BYTES;
  static constexpr int ONES_OFF = K_BYTES + U_BYTES;
  static constexpr int B_OFF = 0;  // two B buffers: segments alternate
  static constexpr int K_OFF = (B_OFF + 2 * B_BYTES + 1023) / 1024 * 1024;
  static constexpr int V_OFF = K_OFF + KST * K_BYTES;
  static constexpr int BAR_OFF = V_OFF + VST * V_STAGE;
  static constexpr int XCH_OFF = BAR_OFF + 256;  // row max [2 blocks][2 halves][BM], then a ticket word
  static constexpr int TOTAL = XCH_OFF + 4 * BM * 4 + 16;
  // TMEM columns: S double buffer; then [O | Z | L], the accumulator of
  // P [V | U | ones] (column 0 of the 16 L columns is the row sum l)
  static constexpr uint32_t COL_S0 = 0, COL_S1 = BN, COL_O = 2 * BN, COL_Z = 2 * BN + D, COL_L = 2 * BN + D + RK;
  static constexpr uint32_t COL_Q = 448;  // the Q tile, bf16 pairs: the A operand of S = Q K^T
  static_assert(2 * BN + D + RK + 16 <= (int)COL_Q && COL_Q + D / 2 <= TMEM_COLS, "TMEM budget");
  static_assert(K_BYTES % 1024 == 0 && V_STAGE % 1024 == 0, "stage alignment");
  static constexpr int REC = BM * (D + 2);  // floats of a partial record: m, l, O + Z B per row
};

struct Bars {
  uint64_t q_full;     // the segment's Q is in TMEM (one arrival per softmax warp); phase = segment
  uint64_t b_full[2];  // B_i,g of segment s has landed in buffer s & 1
  uint64_t b_free[2];  // the epilogue of segment s is done with buffer s & 1 (one arrival per softmax warp)
  uint64_t zb_full;    // Z of the segment is in TMEM as bf16 (one arrival per softmax warp); phase = segment
  uint64_t zb_done;    // O += Z B_i,g of the segment has been computed; phase = segment
  uint64_t k_full[KST];
  uint64_t k_empty[KST];
  uint64_t v_full[VST];
  uint64_t v_empty[VST];
  uint64_t s_full[2];
  uint64_t p_full[2];
  // O/Z/l accumulation of block n (counted over the CTA) completes phase n >> 1
  // of o_ready[n & 1].  With two barriers the block before any awaited one is
  // always already complete, so a parity wait can never be satisfied by a stale phase.
  uint64_t o_ready[2];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  uintptr_t v = reinterpret_cast<uintptr_t>(p);
  return reinterpret_cast<uint8_t*>((v + 1023) & ~uintptr_t(1023));
}


// 128-key blocks of chunk tile tb: the keys any of its rows sees
__device__ __forceinline__ int tile_blocks(const PrefillParams& p, int tb) {
  const int TM = BM / p.G;
  const int j0 = tb * TM;
  const int rows = min(TM, p.T - j0);
  return (p.L0 + j0 + rows + BN - 1) / BN;
}

// One segment of a CTA's range: blocks [lo, hi) of one tile.  Tiles are
// ordered (KV head, agent, chunk tile); flat block index f0 + jb.
struct PSeg {
  int g, agent, tb, j0, nb, lo, hi, tile;
  long long f0;
};

__device__ __forceinline__ PSeg pseg_at(const PrefillParams& p, long long f, long long f_end) {
  PSeg s;
  const long long ga = f / p.W_ga;
  const long long rem = f - ga * p.W_ga;
  long long base = 0;
  int tb = 0;
  for (; tb < p.n_tb - 1; ++tb) {
    const int nb = tile_blocks(p, tb);
    if (rem < base + nb) break;
    base += nb;
  }
  s.agent = (int)(ga % p.N);
  s.g = (int)(ga / p.N);
  s.tb = tb;
  s.tile = (int)ga * p.n_tb + tb;
  s.j0 = tb * (BM / p.G);
  s.nb = tile_blocks(p, tb);
  s.lo = (int)(rem - base);
  const long long hi = s.lo + (f_end - f);
  s.hi = hi < s.nb ? (int)hi : s.nb;
  s.f0 = f - s.lo;
  return s;
}

// CTA owning flat block f when W blocks are split evenly over C CTAs
__device__ __forceinline__ long long pf_owner(long long f, long long W, long long C) { return ((f + 1) * C - 1) / W; }

__device__ __forceinline__ int agent_offset(const PrefillParams& p, int agent, bool flag) {
  if (!p.offsets) return 0;
  const int a = __ldg(p.offsets + agent);
  if (a < 0) {
    if (flag) atomicOr(p.flags, LRKV_DEVFLAG_OFFSET);
    return 0;
  }
  return a;
}

template <int D, int RK>
__global__ void __launch_bounds__(THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmU,
                   const __grid_constant__ CUtensorMap tmB, const PrefillParams p) {
  using Lay = PrefillLayout<D, RK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + Lay::BAR_OFF);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long C = gridDim.x;
  const long long f_begin = (long long)blockIdx.x * p.W / C;
  const long long f_end = (long long)(blockIdx.x + 1) * p.W / C;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 8);
    mbar_init(&bars->zb_full, 8);
    mbar_init(&bars->zb_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->b_full[b], 1);
      mbar_init(&bars->b_free[b], 8);
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 8);  // every softmax warp
      mbar_init(&bars->o_ready[b], 1);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 || warp == 2) {
    // ======================= producers: K and B (warp 0), V and U (warp 2) =======================
    // Separate issuers, so that K blocks run ahead by their own ring depth and
    // never wait behind a V stage that the PV of two blocks back still holds.
    // (With the stall test hook they issue nothing, so the other roles' waits run out.)
    if (lane == 0 && !p.stall) {
      const bool k_role = warp == 0;
      const uint64_t pol_kv = policy_evict_last();  // K/V blocks are reused by the other tiles of the KV head
      const int n_pages = p.page_table ? (p.L0 + p.T + 63) / 64 : 0;
      const int NS = k_role ? KST : VST;
      uint64_t* full = k_role ? bars->k_full : bars->v_full;
      uint64_t* empty = k_role ? bars->k_empty : bars->v_empty;
      int n = 0, si = 0;
      bool ok = true;
      for (long long f = f_begin; f < f_end && ok; ++si) {
        const PSeg sg = pseg_at(p, f, f_end);
        f += sg.hi - sg.lo;
        const int a_i = agent_offset(p, sg.agent, k_role);
        const int u_slot = p.mode == LRKV_BASE_SHARED ? sg.agent : 0;
        if (k_role) {
          // B_i,g of this segment into buffer si & 1, once segment si - 2's epilogue is done with it
          // After an abort the softmax warps release B buffers whose copies may still be
          // landing: issue nothing more (the abort word is read after the wait's acquire).
          if ((si >= 2 && !mbar_wait_bounded(&bars->b_free[si & 1], ((si >> 1) - 1) & 1, abort_flag, p.flags, p.spin_cap, true)) ||
              *abort_flag) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->b_full[si & 1], Lay::B_BYTES);
#pragma unroll
          for (int at = 0; at < D / 64; ++at)  // 128B-swizzled atoms [RK ranks][64 dims]
            tma_load_4d(smem + Lay::B_OFF + (si & 1) * Lay::B_BYTES + at * (RK * 128), &tmB, &bars->b_full[si & 1],
                        at * 64, sg.g, 0, sg.agent, policy_evict_first());
        }
        for (int jb = sg.lo; jb < sg.hi; ++jb, ++n) {
          const int st = n % NS;
          if (!mbar_wait_bounded(&empty[st], ((n / NS) & 1) ^ 1, abort_flag, p.flags, p.spin_cap, true) || *abort_flag) {
            ok = false;
            break;
          }
          int phys[BN / 64];
          if (p.page_table) {
#pragma unroll
            for (int pg = 0; pg < BN / 64; ++pg) {
              int lp = jb * (BN / 64) + pg;
              if (lp >= n_pages) lp = 0;  // past the chunk: any valid page (masked out in the softmax)
              int ph_ = __ldg(p.page_table + (size_t)p.session * p.pt_stride + lp);
              if (ph_ < 0 || ph_ >= p.num_pages) {
                atomicOr(p.flags, LRKV_DEVFLAG_PAGE);
                ph_ = 0;
              }
              phys[pg] = ph_;
            }
          }
          if (k_role) {
            uint8_t* Ks = smem + Lay::K_OFF + st * Lay::K_BYTES;
            mbar_arrive_expect_tx(&full[st], Lay::K_BYTES);
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
              if (!p.page_table) {
                tma_load_4d(Ks + hh * (BN * 128), &tmK, &full[st], hh * 64, jb * BN, sg.g, p.session, pol_kv);
              } else {
#pragma unroll
                for (int pg = 0; pg < BN / 64; ++pg)
                  tma_load_4d(Ks + hh * (BN * 128) + pg * (64 * 128), &tmK, &full[st], hh * 64, 0, sg.g, phys[pg],
                              pol_kv);
              }
            }
          } else {
            const bool need_u = jb * BN + BN > a_i;
            uint8_t* Vs = smem + Lay::V_OFF + st * Lay::V_STAGE;
            uint8_t* Us = Vs + Lay::U_OFF;
            mbar_arrive_expect_tx(&full[st], Lay::K_BYTES + (need_u ? Lay::U_BYTES : 0));
#pragma unroll
            for (int at = 0; at < D / RK; ++at) {  // RK-wide atoms of V, each [BN keys][RK dims]
              if (!p.page_table) {
                tma_load_4d(Vs + at * Lay::U_BYTES, &tmV, &full[st], at * RK, jb * BN, sg.g, p.session, pol_kv);
              } else {
#pragma unroll
                for (int pg = 0; pg < BN / 64; ++pg)
                  tma_load_4d(Vs + at * Lay::U_BYTES + pg * (64 * RK * 2), &tmV, &full[st], at * RK, 0, sg.g,
                              phys[pg], pol_kv);
              }
            }
            if (need_u) tma_load_4d(Us, &tmU, &full[st], 0, jb * BN, u_slot, p.session, pol_kv);
          }
        }
      }
      if (*abort_flag) {
        // let every copy this issuer started land before the CTA can exit
        uint32_t spins = 0;
        if (k_role) {
          for (int sj = si > 2 ? si - 2 : 0; sj < si; ++sj) {
            spins = 0;
            while (!mbar_try_wait(&bars->b_full[sj & 1], (sj >> 1) & 1) && ++spins < kSpinCap) {
            }
          }
        }
        for (int blk = n > NS ? n - NS : 0; blk < n; ++blk) {
          spins = 0;
          while (!mbar_try_wait(&full[blk % NS], (blk / NS) & 1) && ++spins < kSpinCap) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    // Over the CTA's blocks n = 0, 1, ...: S_n, then [O | Z | l] += P_{n-1} [V | U | 1].
    constexpr uint32_t ID_QK = umma_idesc_bf16(BM, BN, 0, 0);
    constexpr uint32_t ID_PVU = umma_idesc_bf16(BM, D + RK + 16, 0, 1);  // [O | Z | l] += P [V | U | 1]
    constexpr uint32_t VU_LAYOUT = RK == 32 ? 4u : 6u;  // 64B / 32B swizzle: atoms of RK bf16 per key row
    constexpr uint32_t VU_LBO = Lay::U_BYTES;           // next atom along d + r
    constexpr uint32_t VU_SBO = 8 * RK * 2;             // next eight key rows
    bool ok = true;
    int n = 0, si = 0;
    // the block awaiting its PV MMA
    bool pv_pending = false;
    int pv_n = 0, pv_jb = 0, pv_a = 0, pv_si = 0;
    bool pv_first = false, pv_last = false;
    constexpr uint32_t ID_ZB = umma_idesc_bf16(BM, D, 0, 1);  // O += Z B_i,g
    auto issue_pv = [&]() -> bool {
      const int st = pv_n % VST;
      if (!mbar_wait_bounded(&bars->p_full[pv_n & 1], (pv_n >> 1) & 1, abort_flag, p.flags, p.spin_cap, true)) return false;
      if (!mbar_wait_bounded(&bars->v_full[st], (pv_n / VST) & 1, abort_flag, p.flags, p.spin_cap, true)) return false;
      uint8_t* Us = smem + Lay::V_OFF + st * Lay::V_STAGE + Lay::U_OFF;
      if (pv_jb * BN < pv_a) {
        // U rows before the offset are zero-filled before the MMA reads them: all
        // of a block wholly before it (its U was not loaded), the head of the block holding it
        const int nz = min(pv_a - pv_jb * BN, BN);  // rows [0, nz)
        uint4* z4 = reinterpret_cast<uint4*>(Us);
        const int n16 = nz * RK * 2 / 16;
        for (int x = lane; x < n16; x += 32) z4[x] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + Lay::V_OFF + st * Lay::V_STAGE);
        const uint32_t a_p = tmem + (pv_n & 1 ? Lay::COL_S1 : Lay::COL_S0);
        // the segment's first block overwrites O, Z and l
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t b = umma_desc(v_base + kk * (16 * RK * 2), VU_LBO, VU_SBO, VU_LAYOUT);
          umma_ts(tmem + Lay::COL_O, a_p + kk * 8, b, ID_PVU, (!pv_first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->v_empty[st]);
        umma_commit(&bars->o_ready[pv_n & 1]);
      }
      __syncwarp();
      if (pv_last) {
        // the segment's O += Z B_i,g: Z (bf16 pairs) in the S buffer of its last block, B in buffer pv_si & 1
        if (!mbar_wait_bounded(&bars->zb_full, pv_si & 1, abort_flag, p.flags, p.spin_cap, true)) return false;
        if (!mbar_wait_bounded(&bars->b_full[pv_si & 1], (pv_si >> 1) & 1, abort_flag, p.flags, p.spin_cap, true)) return false;
        if (lane == 0) {
          tc_fence_after();
          const uint32_t b_base = smem_u32(smem + Lay::B_OFF + (pv_si & 1) * Lay::B_BYTES);
          const uint32_t a_z = tmem + (pv_n & 1 ? Lay::COL_S1 : Lay::COL_S0);
#pragma unroll
          for (int part = 0; part < 2; ++part) {  // Z_hi B, then Z_lo B (columns RK / 2 on)
#pragma unroll
            for (int kk = 0; kk < RK / 16; ++kk) {
              const uint64_t b = umma_desc(b_base + kk * (16 * 128), RK * 128, 1024, 2);
              umma_ts(tmem + Lay::COL_O, a_z + part * (RK / 2) + kk * 8, b, ID_ZB, 1u);
            }
          }
          umma_commit(&bars->zb_done);
        }
        __syncwarp();
      }
      return true;
    };
    for (long long f = f_begin; f < f_end && ok; ++si) {
      const PSeg sg = pseg_at(p, f, f_end);
      f += sg.hi - sg.lo;
      const int a_i = agent_offset(p, sg.agent, false);
      // the segment's Q is in TMEM (its previous content was read by the last S issued)
      ok = mbar_wait_bounded(&bars->q_full, si & 1, abort_flag, p.flags, p.spin_cap, true);
      for (int jb = sg.lo; jb < sg.hi && ok; ++jb, ++n) {
        const int st = n % KST;
        ok = mbar_wait_bounded(&bars->k_full[st], (n / KST) & 1, abort_flag, p.flags, p.spin_cap, true);
        if (!ok) break;
        if (lane == 0) {
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + Lay::K_OFF + st * Lay::K_BYTES);
          const uint32_t d_s = tmem + (n & 1 ? Lay::COL_S1 : Lay::COL_S0);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t b = umma_desc(k_base + (ks >> 2) * (BN * 128) + (ks & 3) * 32, 16, 1024, 2);
            umma_ts(d_s, tmem + Lay::COL_Q + ks * 8, b, ID_QK, ks > 0);
          }
          umma_commit(&bars->s_full[n & 1]);
          umma_commit(&bars->k_empty[st]);
        }
        __syncwarp();
        if (pv_pending && !(ok = issue_pv())) break;
        pv_pending = true;
        pv_n = n;
        pv_jb = jb;
        pv_a = a_i;
        pv_si = si;
        pv_first = jb == sg.lo;
        pv_last = jb == sg.hi - 1;
      }
    }
    if (ok && pv_pending) issue_pv();
  } else if (warp >= 4) {
    // ======================= Q, softmax + epilogue (two warpgroups) =======================
    const int wg = (warp - 4) >> 2;           // key half of every block
    const int row = (warp & 3) * 32 + lane;   // TMEM lane and S/O row
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    constexpr int HB = BN / 2;                // keys per half
    const int c0 = wg * HB;
    float* xmax = reinterpret_cast<float*>(smem + Lay::XCH_OFF);  // [blk & 1][half][row]
    volatile int* ticket_last = reinterpret_cast<volatile int*>(xmax + 4 * BM);
    const int jj = row / p.G, hh = row % p.G;
    // A tile holds floor(128 / G) tokens x G heads; when G does not divide 128
    // the last 128 mod G rows belong to no token: no query, no output.
    const bool row_used = jj < BM / p.G;
    const float NEG_INF = -INFINITY;
    bool ok = true;

    // this row's Q of segment sg into TMEM: half wg of its d dims as bf16 pairs (zeros past the chunk)
    auto load_q = [&](const PSeg& sg) {
      constexpr int QH = D / 2;  // dims per half
      const int token = sg.j0 + jj;
      uint32_t qw[QH / 2];
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(p.q) + (((size_t)sg.agent * p.T + token) * p.Hq + sg.g * p.G + hh) * D +
          wg * QH);
#pragma unroll
      for (int v = 0; v < QH / 8; ++v) {
        const uint4 w = (row_used && token < p.T) ? __ldg(qsrc + v) : make_uint4(0, 0, 0, 0);
        qw[4 * v] = w.x;
        qw[4 * v + 1] = w.y;
        qw[4 * v + 2] = w.z;
        qw[4 * v + 3] = w.w;
      }
      if constexpr (QH / 2 == 32) tmem_st32(tmem + lane_addr + Lay::COL_Q + wg * (QH / 2), qw);
      else tmem_st16(tmem + lane_addr + Lay::COL_Q + wg * (QH / 2), qw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_full);
    };

    if (wg == 1) {
      // the constant atom of every V stage: logical column 0 of each key row is
      // bf16 1.0.  Its rows use the RK-wide swizzle of V and U: 16-byte chunk c
      // of row r sits at chunk c ^ (r >> 1) & 3 (64-byte rows) or c ^ (r >> 2) & 1
      // (32-byte rows).
      constexpr int CPR = RK / 8;  // 16-byte chunks per row
      for (int q = row; q < VST * BN * CPR; q += BM) {
        const int stg = q / (BN * CPR), r = (q / CPR) % BN, pc = q % CPR;
        const int swz = RK == 32 ? (r >> 1) & 3 : (r >> 2) & 1;
        uint4* dst = reinterpret_cast<uint4*>(smem + Lay::V_OFF + stg * Lay::V_STAGE + Lay::ONES_OFF) + r * CPR + pc;
        *dst = make_uint4((pc ^ swz) == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();  // the tensor core reads it through the async proxy
    }
    if (f_begin < f_end) load_q(pseg_at(p, f_begin, f_end));

    // Both warpgroups pass the same named barriers whatever happens: after a
    // failed wait they skip the waits, not the barriers.
    int n = 0, si = 0;
    for (long long f = f_begin; f < f_end; ++si) {
      const PSeg sg = pseg_at(p, f, f_end);
      f += sg.hi - sg.lo;
      const bool has_next = f < f_end;
      const int token = sg.j0 + jj;
      const int limit = p.L0 + token;  // last visible key of this row
      float m_ref = NEG_INF;
      for (int jb = sg.lo; jb < sg.hi; ++jb, ++n) {
        if (ok) ok = mbar_wait_bounded(&bars->s_full[n & 1], (n >> 1) & 1, abort_flag, p.flags, p.spin_cap, true);
        tc_fence_after();
        const uint32_t s_col = n & 1 ? Lay::COL_S1 : Lay::COL_S0;
        float x[HB];
#pragma unroll
        for (int c = 0; c < HB / 32; ++c)
          tmem_ld32(tmem + lane_addr + s_col + c0 + c * 32, reinterpret_cast<uint32_t*>(x) + c * 32);
        tmem_wait_ld();
        // the segment's last S is computed: the next segment's Q may replace this one
        if (jb == sg.hi - 1 && has_next) load_q(pseg_at(p, f, f_end));
        const int key0 = jb * BN + c0;
        if (key0 + HB - 1 > p.L0 + sg.j0) {  // some key of the half is past some row's limit
#pragma unroll
          for (int cc = 0; cc < HB; ++cc) x[cc] = key0 + cc <= limit ? x[cc] : NEG_INF;
        }
        // row max over the half: eight independent chains of three-input maxima, then a
        // tree; then the other half's.  The softmax warps' instruction streams pace this
        // phase, so every instruction saved here shortens the block.
        static_assert(HB % 16 == 8 || HB % 16 == 0, "row-max chains");
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = x[e];
#pragma unroll
        for (int cc = 8; cc + 16 <= HB; cc += 16) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], x[cc + e], x[cc + 8 + e]);
        }
        if constexpr (HB % 16 == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[HB - 8 + e]);
        }
        float* xm = xmax + (n & 1) * 2 * BM;
        xm[wg * BM + row] = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        named_bar_sync(2 + (warp & 3), 64);  // the two warps of these 32 rows; both have read their S columns
        float mx = fmaxf(xm[row], xm[BM + row]);
        mx *= p.scale_log2;  // the scale is positive: the max commutes with it
        const bool need = mx > m_ref + 8.f;
        if (__any_sync(0xffffffffu, need)) {  // the same vote in both halves (same rows, same values)
          const float m_new = fmaxf(m_ref, mx);
          const float alpha = m_new == NEG_INF ? 1.f : fast_exp2(m_ref - m_new);
          if (jb > sg.lo) {
            // O, Z and l hold the segment's blocks before this one: rescale this
            // half's share of their columns in TMEM once the previous PV is done
            if (ok) ok = mbar_wait_bounded(&bars->o_ready[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, p.flags, p.spin_cap, true);
            tc_fence_after();
#pragma unroll
            for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_addr + Lay::COL_O + c * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st32(tmem + lane_addr + Lay::COL_O + c * 32, r);
            }
            if (wg == 1) {  // Z and l: RK + 16 columns
              uint32_t r[32];
              tmem_ld32(tmem + lane_addr + Lay::COL_Z, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st32(tmem + lane_addr + Lay::COL_Z, r);
              if constexpr (RK == 32) {
                tmem_ld16(tmem + lane_addr + Lay::COL_L, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                tmem_st16(tmem + lane_addr + Lay::COL_L, r);
              }
            }
            tmem_wait_st();
          }
          m_ref = m_new;
        }
        const float mu = m_ref == NEG_INF ? 0.f : m_ref;
        // (the row sum l of exactly these bf16 weights is accumulated by the MMA)
        // Two weights' exponent arguments per packed fma (each lane a correctly rounded
        // fma, the same value fmaf gives).
        uint32_t pk[HB / 2];
        unsigned long long ss, mm;  // (scale, scale) and (-mu, -mu)
        asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(p.scale_log2));
        asm("mov.b64 %0, {%1, %1};" : "=l"(mm) : "f"(-mu));
#pragma unroll
        for (int cc = 0; cc < HB / 2; ++cc) {
          unsigned long long xx, aa;
          asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x[2 * cc]), "f"(x[2 * cc + 1]));
          asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(aa) : "l"(xx), "l"(ss), "l"(mm));
          float a0, a1;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(aa));
          pk[cc] = pack_bf16x2(fast_exp2(a0), fast_exp2(a1));
        }
        // P of keys [c0, c0 + 64) as bf16 pairs: TMEM columns s_col + c0 / 2 + [0, 32)
        tmem_st32(tmem + lane_addr + s_col + c0 / 2, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[n & 1]);
      }

      // ---- segment epilogue.  Z goes to TMEM as bf16 (into the S buffer of the
      // last block, free once its PV is done) for the O += Z B_i,g MMA; then
      // out = O / l, or this segment's rows are published for the tile's last CTA.
      const int nl = n - 1;  // the segment's last block
      if (ok) ok = mbar_wait_bounded(&bars->o_ready[nl & 1], (nl >> 1) & 1, abort_flag, p.flags, p.spin_cap, true);
      tc_fence_after();
      float l;
      {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + Lay::COL_Z, r);  // Z, then l when RK = 16
        tmem_wait_ld();
        if constexpr (RK == 16) {
          l = __uint_as_float(r[Lay::COL_L - Lay::COL_Z]);
        } else {
          uint32_t r2[16];
          tmem_ld16(tmem + lane_addr + Lay::COL_L, r2);
          tmem_wait_ld();
          l = __uint_as_float(r2[0]);
        }
        if (wg == 1) {
          // Z = Z_hi + Z_lo with both parts bf16: Z_hi = bf16(Z), Z_lo = bf16(Z - Z_hi)
          // (the difference is exact in fp32), so the two MMAs Z_hi B + Z_lo B carry
          // Z to about 2^-17 of its size instead of the 2^-9 of one bf16 rounding.
          uint32_t zh[RK / 2], zl[RK / 2];
#pragma unroll
          for (int k = 0; k < RK / 2; ++k) {
            const float z0 = __uint_as_float(r[2 * k]), z1 = __uint_as_float(r[2 * k + 1]);
            zh[k] = pack_bf16x2(z0, z1);
            zl[k] = pack_bf16x2(z0 - __uint_as_float(zh[k] << 16), z1 - __uint_as_float(zh[k] & 0xffff0000u));
          }
          const uint32_t zcol = nl & 1 ? Lay::COL_S1 : Lay::COL_S0;
          if constexpr (RK == 32) {
            tmem_st16(tmem + lane_addr + zcol, zh);
            tmem_st16(tmem + lane_addr + zcol + RK / 2, zl);
          } else {
            tmem_st8(tmem + lane_addr + zcol, zh);
            tmem_st8(tmem + lane_addr + zcol + RK / 2, zl);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->zb_full);
      if (ok) ok = mbar_wait_bounded(&bars->zb_done, si & 1, abort_flag, p.flags, p.spin_cap, true);
      tc_fence_after();
      const bool whole = sg.lo == 0 && sg.hi == sg.nb;
      bool finish = true;
      const float* recs = nullptr;  // the tile's partial records, when they are merged here
      int parts = 1;
      float M = NEG_INF;            // the largest record max of this row
      if (!whole) {
        // publish this segment's rows: m, l and this half's columns of O + Z B
        const long long c_first = pf_owner(sg.f0, p.W, C);
        parts = (int)(pf_owner(sg.f0 + sg.nb - 1, p.W, C) - c_first + 1);
        const int slot = (int)((long long)blockIdx.x - c_first);
        float* base = p.partials + (size_t)sg.tile * p.max_parts * Lay::REC;
        float* rec = base + (size_t)slot * Lay::REC;
        if (wg == 0) {
          rec[row] = m_ref;
          rec[BM + row] = l;
        }
#pragma unroll 1
        for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + Lay::COL_O + c * 32, r);
          tmem_wait_ld();
          float* orow = rec + 2 * BM + (size_t)row * D + c * 32;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            __stcg(reinterpret_cast<float4*>(orow + e), make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                                    __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3])));
        }
        __threadfence();
        named_bar_sync(1, SMX_THREADS);
        if (threadIdx.x == 128) {
          const int prev = atomicAdd(p.tickets + sg.tile, 1);
          const int last = prev == parts - 1;
          if (last) p.tickets[sg.tile] = 0;
          *ticket_last = last;
        }
        named_bar_sync(1, SMX_THREADS);
        finish = *ticket_last != 0;
        if (finish) {
          __threadfence();
          recs = base;
          for (int j = 0; j < parts; ++j) M = fmaxf(M, __ldcg(base + (size_t)j * Lay::REC + row));
          l = 0.f;
          for (int j = 0; j < parts; ++j) {
            const float* rj = base + (size_t)j * Lay::REC;
            const float mj = __ldcg(rj + row);
            l += (mj == NEG_INF ? 0.f : fast_exp2(mj - M)) * __ldcg(rj + BM + row);
          }
        }
      }
      if (finish) {
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const bool write = row_used && token < p.T && ok;
        const int h = sg.g * p.G + hh;
#pragma unroll 1
        for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
          float acc[32];
          if (recs == nullptr) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_addr + Lay::COL_O + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(r[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0.f;
            for (int j = 0; j < parts; ++j) {
              const float* rj = recs + (size_t)j * Lay::REC;
              const float mj = __ldcg(rj + row);
              const float w = mj == NEG_INF ? 0.f : fast_exp2(mj - M);
              const float4* orow = reinterpret_cast<const float4*>(rj + 2 * BM + (size_t)row * D + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 v4 = __ldcg(orow + e);
                acc[4 * e] = fmaf(w, v4.x, acc[4 * e]);
                acc[4 * e + 1] = fmaf(w, v4.y, acc[4 * e + 1]);
                acc[4 * e + 2] = fmaf(w, v4.z, acc[4 * e + 2]);
                acc[4 * e + 3] = fmaf(w, v4.w, acc[4 * e + 3]);
              }
            }
          }
          if (write) {
            const size_t oi = (((size_t)sg.agent * p.T + token) * p.Hq + h) * D + c * 32;
            if (p.out_f32) {
              float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(p.out) + oi);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                o4[q4] = make_float4(acc[4 * q4] * inv_l, acc[4 * q4 + 1] * inv_l, acc[4 * q4 + 2] * inv_l,
                                     acc[4 * q4 + 3] * inv_l);
            } else {
              uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + oi);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                o4[q4] = make_uint4(pack_bf16x2(acc[8 * q4] * inv_l, acc[8 * q4 + 1] * inv_l),
                                    pack_bf16x2(acc[8 * q4 + 2] * inv_l, acc[8 * q4 + 3] * inv_l),
                                    pack_bf16x2(acc[8 * q4 + 4] * inv_l, acc[8 * q4 + 5] * inv_l),
                                    pack_bf16x2(acc[8 * q4 + 6] * inv_l, acc[8 * q4 + 7] * inv_l));
            }
          }
        }
      }
      // B buffer si & 1 and the O/Z/l columns are free for the segment after next / the next segment
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->b_free[si & 1]);
    }
  }
  // ---- teardown: every TMEM reader is done before the owner frees it
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, int RK>
lrkv_status launch_t(const PrefillParams& p, const PrefillMaps& m, int grid, cudaStream_t stream) {
  using Lay = PrefillLayout<D, RK>;
  auto kern = prefill_kernel<D, RK>;
  const int smem = Lay::TOTAL + 1024;
  if (ensure_dynamic_smem<prefill_kernel<D, RK>>(smem) != cudaSuccess) return LRKV_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap* t = static_cast<const CUtensorMap*>(m.maps);
  if (cudaLaunchKernelEx(&cfg, kern, t[0], t[1], t[2], t[3], p) != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

}  // namespace

PrefillPlan plan_prefill(int T, int L0, int G, int Hkv, int N, int D, int sms) {
  PrefillPlan pl = {};
  const int TM = BM / G;
  pl.n_tb = (T + TM - 1) / TM;
  pl.tiles = Hkv * N * pl.n_tb;
  long long w = 0;
  int nb_max = 0;
  for (int tb = 0; tb < pl.n_tb; ++tb) {
    const int j0 = tb * TM;
    const int rows = T - j0 < TM ? T - j0 : TM;
    const int nb = (L0 + j0 + rows + BN - 1) / BN;
    w += nb;
    nb_max = nb > nb_max ? nb : nb_max;
  }
  pl.W_ga = w;
  pl.W = w * Hkv * N;
  pl.ctas = (int)(pl.W < sms ? pl.W : sms);
  const long long per = pl.ctas > 0 ? pl.W / pl.ctas : 1;  // fewest blocks a CTA gets
  pl.max_parts = (int)((nb_max + per - 1) / per) + 1;
  pl.tickets_off = kWsHeaderBytes;
  pl.partials_off = (pl.tickets_off + (size_t)pl.tiles * 4 + 255) / 256 * 256;
  pl.bytes = pl.partials_off + (size_t)pl.tiles * pl.max_parts * BM * (D + 2) * 4;
  return pl;
}

int prefill_smem_bytes(int D, int RK) {
  if (D == 128 && RK == 32) return PrefillLayout<128, 32>::TOTAL + 1024;
  if (D == 128 && RK == 16) return PrefillLayout<128, 16>::TOTAL + 1024;
  if (D == 64 && RK == 32) return PrefillLayout<64, 32>::TOTAL + 1024;
  if (D == 64 && RK == 16) return PrefillLayout<64, 16>::TOTAL + 1024;
  return -1;
}

lrkv_status launch_prefill(const PrefillParams& p, const PrefillMaps& m, int D, int RK, int grid, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128 && RK == 32) return launch_t<128, 32>(p, m, grid, st);
  if (D == 128 && RK == 16) return launch_t<128, 16>(p, m, grid, st);
  if (D == 64 && RK == 32) return launch_t<64, 32>(p, m, grid, st);
  if (D == 64 && RK == 16) return launch_t<64, 16>(p, m, grid, st);
  return LRKV_ERR_UNSUPPORTED;
}

}  // namespace lrkv
