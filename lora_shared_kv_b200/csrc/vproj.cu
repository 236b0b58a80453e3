// The value projection with the adapters' down-projections side by side:
//     [V_base | U_1 ... U_n] = X [W0_v | A_1 ... A_n]
// for the T new tokens of a session, written straight into the shared base
// value cache (dense or paged) and the rank-r caches.  Eq. 3 of "LRAgent:
// Efficient KV Cache Sharing for Multi-LoRA LLM Agents" splits agent i's value
// projection as X W0 + (X A_i) B_i; both parts read the same hidden states, so
// one GEMM produces the shared base values and every U_i row at once.
//
// A tcgen05 GEMM over 128-token x BN-column tiles: X (K-major) and W
// (column-major atoms), both 128B-swizzled, stream through a TMA ring in
// 64-wide K steps; fp32 accumulation in TMEM.  An M = 128 MMA from shared
// memory costs about the same for every N up to 256, so BN is 256 when there
// are many tiles.  When there are few, the K loop of a tile is split over a
// thread-block cluster of S CTAs (S <= 8, one K range each) and BN is 128:
// each CTA parks its fp32 partial tile in its own shared memory (the ring is
// idle by then) and, after a cluster barrier, sums one slice of the tile's
// rows over all S partials through distributed shared memory, in rank order
// (so the result does not depend on timing); that traffic, not the MMAs,
// bounds a split tile, and it halves with BN.  The sums are converted to bf16
// and each row's columns scattered to its cache: column c < Hkv d goes to KV
// head c / d of the base value cache, the rest to agent slot (c - Hkv d) / r.
// The summation order inside the tensor core is not specified, so U rows made
// here are not bit-identical to the fixed-order append.
#include "common.cuh"
#include "lrkv_internal.h"

namespace lrkv {

namespace {

constexpr int VP_BM = 128;                      // tokens per tile (TMEM lanes)
constexpr int VP_BK = 64;                       // K per stage
constexpr int VP_THREADS = 256;
constexpr int VP_X_BYTES = VP_BM * VP_BK * 2;   // 16 KB
constexpr int VP_ATOM_BYTES = VP_BK * 128;      // 8 KB: 64 k-rows x 128 B
constexpr int VP_RING = 192 * 1024;             // shared memory for the ring
constexpr int VP_SMEM = VP_RING + 256;
constexpr int VP_MAX_ST = 6;
constexpr int VP_MAX_SPLIT = 8;                 // portable cluster size

// A tile of 128 tokens x BN columns (BN = 256, or 128 when the K loop is split:
// each CTA's partial tile, which the split moves across the cluster, halves).
template <int BN>
struct VpTile {
  static constexpr int ATOMS = BN / 64;                            // 64-column W atoms per stage
  static constexpr int STAGE = VP_X_BYTES + ATOMS * VP_ATOM_BYTES;  // 32 or 48 KB
  static constexpr int ST = VP_RING / STAGE;                        // 6 or 4 stages
  static constexpr int RP = BN + 4;  // fp32 pitch of a partial-tile row: conflict-free 16-byte stores
  static_assert(ST <= VP_MAX_ST, "barrier slots");
  static_assert(VP_BM * RP * 4 <= VP_RING, "the partial tile reuses the ring");
};

// Thread-block clusters: distributed shared memory.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Executed by every thread of every CTA of the cluster (warp-converged):
// shared-memory writes made before it are visible cluster-wide after it.  A
// launch without clusters is a cluster of one CTA.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of this CTA's shared address `smem_addr` in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

struct VpBars {
  uint64_t full[VP_MAX_ST];
  uint64_t empty[VP_MAX_ST];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
  int ok;  // this CTA's partial tile is complete
};

template <int BN>
__global__ void __launch_bounds__(VP_THREADS, 1)
    vproj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const VprojParams p) {
  using Sh = VpTile<BN>;
  constexpr int VP_ST = Sh::ST;
  constexpr int VP_STAGE = Sh::STAGE;
  constexpr int VP_RP = Sh::RP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  VpBars* bars = reinterpret_cast<VpBars*>(smem + VP_RING);
  float* part = reinterpret_cast<float*>(smem);  // [VP_BM][VP_RP] once the K loop is done
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * VP_BM;  // first token
  const int n0 = blockIdx.y * BN;  // first output column
  const int S = gridDim.z;            // K split = cluster size; cluster dims (1, 1, S)
  const int z = (int)cluster_ctarank();
  const int nk_all = (p.Dm + VP_BK - 1) / VP_BK;
  const int kt0 = (int)((long long)z * nk_all / S);
  const int nk = (int)((long long)(z + 1) * nk_all / S) - kt0;  // >= 1: the launcher keeps S <= nk_all
  const int natoms = min(Sh::ATOMS, (p.ncols - n0 + 63) / 64);   // W atoms that reach into the weights

  if (threadIdx.x == 0) {
    for (int s = 0; s < VP_ST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    bars->abort_flag = 0;
    bars->ok = 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, BN);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---- TMA producer: this CTA's K steps kt0 .. kt0 + nk - 1
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // W tiles are read by every token tile
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int st = j % VP_ST;
        if (!mbar_wait_bounded(&bars->empty[st], ((j / VP_ST) & 1) ^ 1, abort_flag, p.flags)) break;
        issued = j + 1;
        uint8_t* xs = smem + st * VP_STAGE;
        uint8_t* ws = xs + VP_X_BYTES;
        const int k = (kt0 + j) * VP_BK;
        mbar_arrive_expect_tx(&bars->full[st], VP_X_BYTES + natoms * VP_ATOM_BYTES);
        tma_load_4d(xs, &tmX, &bars->full[st], k, m0, 0, 0, pol);
        for (int at = 0; at < natoms; ++at)
          tma_load_4d(ws + at * VP_ATOM_BYTES, &tmW, &bars->full[st], n0 + at * 64, k, 0, 0, pol);
      }
      if (*abort_flag) {
        for (int j = issued > VP_ST ? issued - VP_ST : 0; j < issued; ++j) {
          uint32_t spins = 0;
          while (!mbar_try_wait(&bars->full[j % VP_ST], (j / VP_ST) & 1) && ++spins < kSpinCap) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: D[128 tokens x 256 columns] += X[tokens, k] W[k, columns]
    // (atoms past the weights' last column are not loaded; their columns are never read)
    constexpr uint32_t ID = umma_idesc_bf16(VP_BM, BN, 0, 1);
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      const int st = j % VP_ST;
      ok = mbar_wait_bounded(&bars->full[st], (j / VP_ST) & 1, abort_flag, p.flags);
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t xs = smem_u32(smem + st * VP_STAGE);
        const uint32_t ws = xs + VP_X_BYTES;
#pragma unroll
        for (int ks = 0; ks < VP_BK / 16; ++ks) {
          const uint64_t a = umma_desc(xs + ks * 32, 16, 1024, 2);                // K-major, 128B swizzle
          const uint64_t b = umma_desc(ws + ks * 2048, VP_ATOM_BYTES, 1024, 2);   // column-major atoms
          umma_ss(tmem, a, b, ID, (j > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars->empty[st]);
        if (j == nk - 1) umma_commit(&bars->acc_full);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ---- the partial tile, one token row per thread (TMEM lane), into shared memory
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const bool ok = mbar_wait_bounded(&bars->acc_full, 0, abort_flag, p.flags);
    tc_fence_after();
    if (!ok) {
      bars->ok = 0;
    } else {
      const int nch = (min(BN, p.ncols - n0) + 31) / 32;
      float4* dst = reinterpret_cast<float4*>(part + row * VP_RP);
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[c * 8 + q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                       __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      }
    }
    tc_fence_before();
  }
  __syncwarp();
  cluster_sync();  // every partial tile of the cluster is in place

  // ---- rows [row_lo, row_hi) of the tile: the sum of the S partials, a warp per
  // two rows at a time, 4 columns per lane in each 128-column half, written as
  // bf16 to the caches
  {
    constexpr int NH = BN / 128;
    int all_ok = 1;
    for (int q = 0; q < S; ++q) all_ok &= ld_cluster_s32(cluster_map(smem_u32(&bars->ok), (uint32_t)q));
    const int row_lo = z * VP_BM / S, row_hi = min((z + 1) * VP_BM / S, p.T - m0);
    auto dest = [&](int row, int c) -> uint16_t* {  // where column c of the tile's row goes (or null)
      const int pos = p.start_row + m0 + row;
      const int hd = p.Hkv * p.d;
      if (c < hd) {
        if (p.page_table) {
          const int pg = __ldg(p.page_table + (size_t)p.session * p.pt_stride + pos / p.page_size);
          if (pg < 0 || pg >= p.num_pages) {
            if (c == 0) atomicOr(p.flags, LRKV_DEVFLAG_PAGE);
            return nullptr;
          }
          return p.v + (size_t)pg * p.v_sp + (size_t)(pos % p.page_size) * p.v_st + (size_t)(c / p.d) * p.v_sh + c % p.d;
        }
        return p.v + (size_t)p.session * p.v_ss + (size_t)pos * p.v_st + (size_t)(c / p.d) * p.v_sh + c % p.d;
      }
      if (c >= p.ncols) return nullptr;
      const int cu = c - hd;
      return p.u + (size_t)p.session * p.u_ss + (size_t)(cu / p.r) * p.u_sa + (size_t)pos * p.u_st + cu % p.r;
    };
    for (int r0 = row_lo + warp; all_ok && r0 < row_hi; r0 += 2 * (VP_THREADS / 32)) {
      const int nr = r0 + VP_THREADS / 32 < row_hi ? 2 : 1;
      float4 acc[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = r0 + h * (VP_THREADS / 32);
        if (h < nr) {
          const uint32_t src = smem_u32(part + row * VP_RP + 4 * lane);
          float4 lo[VP_MAX_SPLIT], hi[VP_MAX_SPLIT];
#pragma unroll
          for (int q = 0; q < VP_MAX_SPLIT; ++q) {
            if (q < S) {
              const uint32_t a = cluster_map(src, (uint32_t)q);
              lo[q] = ld_cluster_f4(a);
              if constexpr (NH == 2) hi[q] = ld_cluster_f4(a + 128 * 4);  // past ncols: never stored
            }
          }
          acc[h][0] = lo[0];
          if constexpr (NH == 2) acc[h][1] = hi[0];
#pragma unroll
          for (int q = 1; q < VP_MAX_SPLIT; ++q) {
            if (q < S) {
              acc[h][0].x += lo[q].x; acc[h][0].y += lo[q].y; acc[h][0].z += lo[q].z; acc[h][0].w += lo[q].w;
              if constexpr (NH == 2) {
                acc[h][1].x += hi[q].x; acc[h][1].y += hi[q].y; acc[h][1].z += hi[q].z; acc[h][1].w += hi[q].w;
              }
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h < nr) {
          const int row = r0 + h * (VP_THREADS / 32);
#pragma unroll
          for (int e = 0; e < NH; ++e) {
            uint16_t* dst = dest(row, n0 + 4 * lane + 128 * e);
            if (dst)
              *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[h][e].x, acc[h][e].y),
                                                          pack_bf16x2(acc[h][e].z, acc[h][e].w));
          }
        }
      }
    }
  }
  __syncwarp();
  cluster_sync();  // the other CTAs have finished reading this CTA's partial tile
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// Largest K split S <= cap whose clusters all fit on the device at once for
// `tiles` tiles (queried once per device, tile width and S; -1 records a failed query).
template <int BN>
int pick_split(int tiles, int cap) {
  constexpr int kDevices = 64;
  static std::atomic<int> cache[kDevices][VP_MAX_SPLIT + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return 1;
  for (int S = cap; S > 1; --S) {
    int n = cache[dev][S].load(std::memory_order_relaxed);
    if (n == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, 1, S);
      cfg.blockDim = dim3(VP_THREADS);
      cfg.dynamicSmemBytes = VP_SMEM + 1024;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = S;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, vproj_kernel<BN>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = -1;
      }
      cache[dev][S].store(n, std::memory_order_relaxed);
    }
    if (tiles <= n) return S;
  }
  return 1;
}

template <int BN>
lrkv_status launch_t(const VprojParams& p, const void* tmX, const void* tmW, int sms, void* stream) {
  const int smem = VP_SMEM + 1024;
  if (ensure_dynamic_smem<vproj_kernel<BN>>(smem) != cudaSuccess) return LRKV_ERR_CUDA;
  const int tiles = ((p.T + VP_BM - 1) / VP_BM) * ((p.ncols + BN - 1) / BN);
  const int nk = (p.Dm + VP_BK - 1) / VP_BK;
  int cap = sms / tiles;
  cap = cap < VP_MAX_SPLIT ? cap : VP_MAX_SPLIT;
  cap = cap < nk ? cap : nk;
  const int S = cap > 1 ? pick_split<BN>(tiles, cap) : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.T + VP_BM - 1) / VP_BM, (p.ncols + BN - 1) / BN, S);
  cfg.blockDim = dim3(VP_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = S;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, vproj_kernel<BN>, *static_cast<const CUtensorMap*>(tmX),
                         *static_cast<const CUtensorMap*>(tmW), p) != cudaSuccess)
    return LRKV_ERR_CUDA;
  return LRKV_OK;
}

}  // namespace

int vproj_smem_bytes() { return VP_SMEM + 1024; }

lrkv_status launch_vproj(const VprojParams& p, const void* tmX, const void* tmW, int sms, void* stream) {
  // 128-column tiles when there are few enough of them that the K loop gets split
  // (half the partial tile to move per CTA), else 256 (half the MMAs per column)
  const int tiles128 = ((p.T + VP_BM - 1) / VP_BM) * ((p.ncols + 127) / 128);
  if (tiles128 * 2 <= sms) return launch_t<128>(p, tmX, tmW, sms, stream);
  return launch_t<256>(p, tmX, tmW, sms, stream);
}

}  // namespace lrkv
