// The value projection with the adapters' down-projections side by side:
//     [V_base | U_1 ... U_n] = X [W0_v | A_1 ... A_n]
// for the T new tokens of a session, written straight into the shared base
// value cache (dense or paged) and the rank-r caches.  Eq. 3 of "LRAgent:
// Efficient KV Cache Sharing for Multi-LoRA LLM Agents" splits agent i's value
// projection as X W0 + (X A_i) B_i; both parts read the same hidden states, so
// one GEMM produces the shared base values and every U_i row at once.
//
// A tcgen05 GEMM: one CTA per 128-token x BN-column tile (BN = 128, or 64 when
// 128-wide tiles would leave SMs idle), K in 64-wide steps through a TMA ring
// of 6 or 8 stages (X K-major, W column-major atoms, both 128B swizzled), fp32
// accumulation in TMEM, and an epilogue that converts to bf16
// and scatters each row's columns to its cache: column c < Hkv d goes to KV
// head c / d of the base value cache, the rest to agent slot (c - Hkv d) / r.
// The summation order inside the tensor core is not specified, so U rows made
// here are not bit-identical to the fixed-order append.
#include "common.cuh"
#include "lrkv_internal.h"

namespace lrkv {

namespace {

constexpr int VP_BM = 128;     // tokens per tile (TMEM lanes)
constexpr int VP_BK = 64;      // K per stage
constexpr int VP_THREADS = 256;
constexpr int VP_X_BYTES = VP_BM * VP_BK * 2;   // 16 KB
constexpr int VP_RING = 192 * 1024;             // shared memory for the ring

template <int BN>
struct VpShape {
  static constexpr int W_BYTES = VP_BK * BN * 2;  // BN / 64 atoms of 64 k-rows x 64 columns
  static constexpr int STAGE = VP_X_BYTES + W_BYTES;
  static constexpr int ST = VP_RING / STAGE;      // 6 (BN = 128) or 8 (BN = 64) stages
  static constexpr int SMEM = ST * STAGE + 256;
};

struct VpBars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

template <int BN>
__global__ void __launch_bounds__(VP_THREADS, 1)
    vproj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const VprojParams p) {
  constexpr int VP_ST = VpShape<BN>::ST;
  constexpr int VP_STAGE = VpShape<BN>::STAGE;
  constexpr int VP_BN = BN;
  static_assert(VP_ST <= 8, "barrier slots");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  VpBars* bars = reinterpret_cast<VpBars*>(smem + VP_ST * VP_STAGE);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * VP_BM;  // first token
  const int n0 = blockIdx.y * VP_BN;  // first output column
  const int nk = (p.Dm + VP_BK - 1) / VP_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < VP_ST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, VP_BN);
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
    // ---- TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // W tiles are read by every token tile
      int issued = 0;
      for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % VP_ST;
        if (!mbar_wait_bounded(&bars->empty[st], ((kt / VP_ST) & 1) ^ 1, abort_flag, p.flags)) break;
        issued = kt + 1;
        uint8_t* xs = smem + st * VP_STAGE;
        uint8_t* ws = xs + VP_X_BYTES;
        mbar_arrive_expect_tx(&bars->full[st], VP_STAGE);
        tma_load_4d(xs, &tmX, &bars->full[st], kt * VP_BK, m0, 0, 0, pol);
#pragma unroll
        for (int at = 0; at < BN / 64; ++at)
          tma_load_4d(ws + at * (VP_BK * 128), &tmW, &bars->full[st], n0 + at * 64, kt * VP_BK, 0, 0, pol);
      }
      if (*abort_flag) {
        for (int kt = issued > VP_ST ? issued - VP_ST : 0; kt < issued; ++kt) {
          uint32_t spins = 0;
          while (!mbar_try_wait(&bars->full[kt % VP_ST], (kt / VP_ST) & 1) && ++spins < kSpinCap) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: D[128 tokens x 128 columns] += X[tokens, k] W[k, columns]
    constexpr uint32_t ID = umma_idesc_bf16(VP_BM, VP_BN, 0, 1);
    bool ok = true;
    for (int kt = 0; kt < nk && ok; ++kt) {
      const int st = kt % VP_ST;
      ok = mbar_wait_bounded(&bars->full[st], (kt / VP_ST) & 1, abort_flag, p.flags);
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t xs = smem_u32(smem + st * VP_STAGE);
        const uint32_t ws = xs + VP_X_BYTES;
#pragma unroll
        for (int ks = 0; ks < VP_BK / 16; ++ks) {
          const uint64_t a = umma_desc(xs + ks * 32, 16, 1024, 2);                 // K-major, 128B swizzle
          const uint64_t b = umma_desc(ws + ks * 2048, VP_BK * 128, 1024, 2);     // column-major atoms
          umma_ss(tmem, a, b, ID, (kt > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars->empty[st]);
        if (kt == nk - 1) umma_commit(&bars->acc_full);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ---- epilogue: one token row per thread (TMEM lane), bf16 into the caches
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const bool ok = mbar_wait_bounded(&bars->acc_full, 0, abort_flag, p.flags);
    tc_fence_after();
    const int t = m0 + row;
    const int pos = p.start_row + t;  // cache row
    const int hd = p.Hkv * p.d;
    uint16_t* vrow = nullptr;         // this token's row of the base value cache, head 0
    if (ok && t < p.T) {
      if (p.page_table) {
        const int pg = __ldg(p.page_table + (size_t)p.session * p.pt_stride + pos / p.page_size);
        if (pg >= 0 && pg < p.num_pages)
          vrow = p.v + (size_t)pg * p.v_sp + (size_t)(pos % p.page_size) * p.v_st;
        else
          atomicOr(p.flags, LRKV_DEVFLAG_PAGE);
      } else {
        vrow = p.v + (size_t)p.session * p.v_ss + (size_t)pos * p.v_st;
      }
    }
#pragma unroll 1
    for (int c = 0; c < VP_BN / 32; ++c) {
      const int c0 = n0 + c * 32;  // first column of the chunk
      if (c0 >= p.ncols) break;
      uint32_t r[32];
      tmem_ld32(tmem + lane_addr + c * 32, r);
      tmem_wait_ld();
      if (!ok || t >= p.T) continue;
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
      if (c0 < hd) {
        // 32 columns of one KV head (d is a multiple of 32)
        if (vrow) {
          uint4* dst = reinterpret_cast<uint4*>(vrow + (size_t)(c0 / p.d) * p.v_sh + c0 % p.d);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      } else {
        // rank columns: agent slots of r columns each (r in {8, 16, 32} divides 32)
        for (int e = 0; e < 32; e += p.r) {
          const int cu = c0 + e - hd;
          if (cu >= p.n_u * p.r) break;
          uint16_t* urow = p.u + (size_t)p.session * p.u_ss + (size_t)(cu / p.r) * p.u_sa + (size_t)pos * p.u_st;
          uint4* dst = reinterpret_cast<uint4*>(urow);
          for (int q = 0; q < p.r / 8; ++q)
            dst[q] = make_uint4(pk[e / 2 + 4 * q], pk[e / 2 + 4 * q + 1], pk[e / 2 + 4 * q + 2], pk[e / 2 + 4 * q + 3]);
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, VP_BN);
  }
}

}  // namespace

int vproj_smem_bytes() { return VpShape<128>::SMEM + 1024; }

lrkv_status launch_vproj(const VprojParams& p, const void* tmX, const void* tmW, int sms, void* stream) {
  // 128-wide tiles, unless they would leave more than half of the SMs idle
  const long long tiles128 = (long long)((p.T + VP_BM - 1) / VP_BM) * ((p.ncols + 127) / 128);
  const bool narrow = tiles128 * 2 <= sms;
  const int bn = narrow ? 64 : 128;
  const int smem = (narrow ? VpShape<64>::SMEM : VpShape<128>::SMEM) + 1024;
  auto kern = narrow ? vproj_kernel<64> : vproj_kernel<128>;
  if ((narrow ? ensure_dynamic_smem<vproj_kernel<64>>(smem) : ensure_dynamic_smem<vproj_kernel<128>>(smem)) !=
      cudaSuccess)
    return LRKV_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.T + VP_BM - 1) / VP_BM, (p.ncols + bn - 1) / bn);
  cfg.blockDim = dim3(VP_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, *static_cast<const CUtensorMap*>(tmX), *static_cast<const CUtensorMap*>(tmW),
                         p) != cudaSuccess)
    return LRKV_ERR_CUDA;
  return LRKV_OK;
}

}  // namespace lrkv
