// Low-rank cache append: U_i[t + shift, :] = X[t, :] A_i for the rows t of
// each agent's range: a contiguous block of new tokens for every agent, or
// per-agent ranges (the tokens each agent has not processed yet).
//
// The rank-r cache X A_i is the adapter half of the split value projection
// (Eq. 3 of "LRAgent: Efficient KV Cache Sharing for Multi-LoRA LLM Agents");
// Fig. 3 of that page appends it for the tokens an agent has not processed yet.
//
// Numerics are a fixed contract so that the result is bit-determined:
// acc = +0.0f, then acc = fmaf(x[t,k], a[k,j], acc) for k = 0, 1, ..., Dm-1 in
// that order, then round-to-nearest-even to bf16.  Tensor cores are not used on
// purpose: their summation order inside an MMA is not specified.  The work is
// tiny next to the attention (T x Dm x r per agent) and runs on the CUDA cores.
#include "common.cuh"

namespace lrkv {

namespace {

// A warp owns 32 consecutive tokens (one per lane) and a group of 8 columns:
// each thread runs 8 independent fmaf chains.  Per k a lane reads its own
// x[t, k] (a conflict-free 32-bit load) and the group's 8 A values (two
// 128-bit loads every lane shares: broadcasts), so shared memory serves 8
// FMAs per lane with 3 loads.  A block of 4 warps covers TB tokens x all r
// columns of one agent; X (transposed, k-major) and A are staged as fp32 one
// k-chunk at a time, the next chunk's global loads held in registers while the
// current chunk is consumed.  Each output still sums k = 0 .. Dm-1 in order.
constexpr int APP_THREADS = 128;
constexpr int KC = 64;  // k per chunk

// The x rows of each agent of one launch (agent agent_base + blockIdx.y):
// block x covers rows begin + TB * blockIdx.x ..; U row = x row + u_shift.
struct AppendRows {
  int begin[kMaxAgents];
  int end[kMaxAgents];
  int agent_base;
  int u_shift;
};

template <int R>
struct AppShape {
  static constexpr int CG = R / 8;                      // column groups of 8
  static constexpr int TB = (APP_THREADS / 32) / CG * 32;  // tokens per block
  static constexpr int XS = TB + 1;                     // padded k-row of the transposed X chunk
  static constexpr int XL = TB * KC / APP_THREADS;      // X loads per thread per chunk
  static constexpr int AL = KC * R / APP_THREADS;       // A loads per thread per chunk
  static_assert(APP_THREADS % KC == 0 && (TB * KC) % APP_THREADS == 0 && (KC * R) % APP_THREADS == 0, "shape");
};

template <int R>
__global__ void __launch_bounds__(APP_THREADS)
    append_kernel_generic(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a, const AppendRows rows,
                          int Dm, __nv_bfloat16* __restrict__ u, long long u_ss, long long u_sa, long long u_st,
                          int session) {
  using S = AppShape<R>;
  __shared__ float xs[KC * S::XS];                // xs[k * XS + token]
  __shared__ __align__(16) float as[KC * R];      // as[k * R + column]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = warp % S::CG;                    // this warp's 8 columns: [8 cg, 8 cg + 8)
  const int tl = (warp / S::CG) * 32 + lane;      // this thread's token within the block
  const int agent = rows.agent_base + blockIdx.y;
  const int T = rows.end[blockIdx.y];
  const int t0 = rows.begin[blockIdx.y] + blockIdx.x * S::TB;
  if (t0 >= T) return;  // past this agent's range (block-uniform)
  const uint16_t* a_ag = a + (size_t)agent * Dm * R;

  // staging: chunk element e = tid + i * APP_THREADS of X sits at token e / KC,
  // k e % KC; as APP_THREADS is a multiple of KC a thread's k is fixed
  constexpr int RSTEP = APP_THREADS / KC;
  const int my_kk = tid % KC, my_row = tid / KC;
  const uint16_t* xp = x + (size_t)(t0 + my_row) * Dm + my_kk;
  uint16_t xr[S::XL], ar[S::AL];
  auto load_chunk = [&](int k0) {
    const bool k_ok = k0 + my_kk < Dm;
#pragma unroll
    for (int i = 0; i < S::XL; ++i)
      xr[i] = (k_ok && t0 + my_row + i * RSTEP < T) ? __ldg(xp + (size_t)i * RSTEP * Dm + k0) : (uint16_t)0;
#pragma unroll
    for (int i = 0; i < S::AL; ++i) {
      const int e = tid + i * APP_THREADS;
      ar[i] = (k0 + e / R < Dm) ? __ldg(a_ag + (size_t)k0 * R + e) : (uint16_t)0;
    }
  };
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  const float* xcol = xs + tl;
  const float4* acol = reinterpret_cast<const float4*>(as + cg * 8);
  load_chunk(0);
  for (int k0 = 0; k0 < Dm; k0 += KC) {
    __syncthreads();  // the previous chunk's reads are done
#pragma unroll
    for (int i = 0; i < S::XL; ++i) xs[my_kk * S::XS + my_row + i * RSTEP] = __uint_as_float((uint32_t)xr[i] << 16);
#pragma unroll
    for (int i = 0; i < S::AL; ++i) as[tid + i * APP_THREADS] = __uint_as_float((uint32_t)ar[i] << 16);
    __syncthreads();
    if (k0 + KC < Dm) load_chunk(k0 + KC);
    const int kc = min(KC, Dm - k0);
    if (kc == KC) {
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        const float xv = xcol[kk * S::XS];
        const float4 a0 = acol[kk * (R / 4)], a1 = acol[kk * (R / 4) + 1];
        acc[0] = fmaf(xv, a0.x, acc[0]);
        acc[1] = fmaf(xv, a0.y, acc[1]);
        acc[2] = fmaf(xv, a0.z, acc[2]);
        acc[3] = fmaf(xv, a0.w, acc[3]);
        acc[4] = fmaf(xv, a1.x, acc[4]);
        acc[5] = fmaf(xv, a1.y, acc[5]);
        acc[6] = fmaf(xv, a1.z, acc[6]);
        acc[7] = fmaf(xv, a1.w, acc[7]);
      }
    } else {
      for (int kk = 0; kk < kc; ++kk) {
        const float xv = xcol[kk * S::XS];
        const float4 a0 = acol[kk * (R / 4)], a1 = acol[kk * (R / 4) + 1];
        acc[0] = fmaf(xv, a0.x, acc[0]);
        acc[1] = fmaf(xv, a0.y, acc[1]);
        acc[2] = fmaf(xv, a0.z, acc[2]);
        acc[3] = fmaf(xv, a0.w, acc[3]);
        acc[4] = fmaf(xv, a1.x, acc[4]);
        acc[5] = fmaf(xv, a1.y, acc[5]);
        acc[6] = fmaf(xv, a1.z, acc[6]);
        acc[7] = fmaf(xv, a1.w, acc[7]);
      }
    }
  }
  const int t = t0 + tl;
  if (t < T) {
    __nv_bfloat16* dst = u + (size_t)session * u_ss + (size_t)agent * u_sa + (size_t)(t + rows.u_shift) * u_st + cg * 8;
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[c] = __float2bfloat16_rn(acc[c]);
  }
}

template <int R>
void launch_generic(const void* x, const void* a, const AppendRows& rows, int n, int max_len, int Dm, void* u,
                    long long u_ss, long long u_sa, long long u_st, int session, cudaStream_t stream) {
  dim3 grid((max_len + AppShape<R>::TB - 1) / AppShape<R>::TB, n);
  append_kernel_generic<R><<<grid, APP_THREADS, 0, stream>>>(static_cast<const uint16_t*>(x),
                                                             static_cast<const uint16_t*>(a), rows, Dm,
                                                             static_cast<__nv_bfloat16*>(u), u_ss, u_sa, u_st,
                                                             session);
}

// ---------------------------------------------------------------------------
// Fast path (Dm a multiple of 8, x and a 16-byte aligned): a warp owns 32
// tokens (one per lane) x 4 columns, so a lane runs 4 fmaf chains and a block
// of 4 warps covers 32 tokens x 16 columns (64 x 8 when r = 8).  X and A
// k-chunks of 128 stream through a cp.async ring deep enough (12 stages, 6 for
// 64-token blocks) that the whole of a 2048-wide hidden state is requested at
// the start: the chunks' global latency overlaps the chains instead of
// stalling them.  A lane reads 8 k of its token's X row with one 128-bit load
// (rows padded to 272 B: conflict-free) and each k's 4 A values (converted to
// fp32 once per chunk) with one broadcast load.
// ---------------------------------------------------------------------------
constexpr int F_KC = 128;       // k per chunk
constexpr int F_XP = F_KC + 8;  // X row pitch in bf16 (272 B)

template <int R>
struct FastShape {
  static constexpr int CGB = R / 4 < 4 ? R / 4 : 4;  // 4-column groups per block
  static constexpr int TGB = 4 / CGB;                 // 32-token groups per block
  static constexpr int TB = 32 * TGB;                 // tokens per block
  static constexpr int CB = 4 * CGB;                  // columns per block
  static constexpr int NCB = R / CB;                  // column blocks
  static constexpr int NS = TB == 32 ? 12 : 6;        // ring stages
  static constexpr int XCP = TB * (F_KC / 8);         // 16-byte X copies per chunk
  static constexpr int ACP = F_KC * CB / 8;           // 16-byte A copies per chunk
  static constexpr int X_STAGE = TB * F_XP;           // bf16 elements
  static constexpr int A_STAGE = F_KC * CB;           // bf16 elements
  static constexpr int SMEM = NS * (X_STAGE + A_STAGE) * 2 + F_KC * CB * 4;
  static_assert(XCP % APP_THREADS == 0 && ACP % APP_THREADS == 0 && (F_KC * CB) % APP_THREADS == 0, "shape");
};

template <int R>
__global__ void __launch_bounds__(APP_THREADS)
    append_kernel_fast(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a, const AppendRows rows, int Dm,
                       __nv_bfloat16* __restrict__ u, long long u_ss, long long u_sa, long long u_st, int session) {
  using S = FastShape<R>;
  constexpr int NS = S::NS;
  extern __shared__ __align__(16) uint8_t app_smem[];
  uint16_t* xr = reinterpret_cast<uint16_t*>(app_smem);            // [NS][TB * F_XP]
  uint16_t* ar = xr + NS * S::X_STAGE;                             // [NS][F_KC * CB]
  float* af = reinterpret_cast<float*>(ar + NS * S::A_STAGE);      // [F_KC * CB]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = warp % S::CGB;
  const int tl = (warp / S::CGB) * 32 + lane;  // token within the block
  const int agent = rows.agent_base + blockIdx.y;
  const int T = rows.end[blockIdx.y];
  const int t0 = rows.begin[blockIdx.y] + blockIdx.x * S::TB;
  if (t0 >= T) return;  // past this agent's range (block-uniform)
  const int c0 = blockIdx.z * S::CB;           // first column of the block
  const uint16_t* a_ag = a + (size_t)agent * Dm * R;
  const int n_chunks = (Dm + F_KC - 1) / F_KC;

  auto issue = [&](int c) {
    if (c < n_chunks) {
      const int k0 = c * F_KC, st = c % NS;
#pragma unroll
      for (int i = 0; i < S::XCP / APP_THREADS; ++i) {
        const int e = tid + i * APP_THREADS;
        const int row = e / (F_KC / 8), seg = e % (F_KC / 8);
        const bool ok = t0 + row < T && k0 + seg * 8 < Dm;
        const uint16_t* src = ok ? x + (size_t)(t0 + row) * Dm + k0 + seg * 8 : x;
        cp_async16(&xr[st * S::X_STAGE + row * F_XP + seg * 8], src, ok ? 16u : 0u);
      }
#pragma unroll
      for (int i = 0; i < S::ACP / APP_THREADS; ++i) {
        const int e = tid + i * APP_THREADS;
        const int row = e / (S::CB / 8), seg = e % (S::CB / 8);
        const bool ok = k0 + row < Dm;
        const uint16_t* src = ok ? a_ag + (size_t)(k0 + row) * R + c0 + seg * 8 : a_ag;
        cp_async16(&ar[st * S::A_STAGE + row * S::CB + seg * 8], src, ok ? 16u : 0u);
      }
    }
    cp_async_commit();  // one group per chunk index, empty past the end
  };

  float acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
#pragma unroll 1
  for (int c = 0; c < NS - 1; ++c) issue(c);
  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<NS - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();          // everyone's; and chunk c - 1 is no longer read
    const int st = c % NS;
#pragma unroll
    for (int i = 0; i < F_KC * S::CB / APP_THREADS; ++i) {
      const int e = tid + i * APP_THREADS;
      af[e] = __uint_as_float((uint32_t)ar[st * S::A_STAGE + e] << 16);
    }
    __syncthreads();
    issue(c + NS - 1);  // into the stage chunk c - 1 used
    const int kc = min(F_KC, Dm - c * F_KC);  // a multiple of 8
    const uint4* xrow = reinterpret_cast<const uint4*>(&xr[st * S::X_STAGE + tl * F_XP]);
    const float4* acol = reinterpret_cast<const float4*>(af) + cg;
    for (int k8 = 0; k8 < kc / 8; ++k8) {
      const uint4 xv = xrow[k8];
      const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float xf = __uint_as_float(q & 1 ? (w[q >> 1] & 0xffff0000u) : (w[q >> 1] << 16));
        const float4 av = acol[(k8 * 8 + q) * (S::CB / 4)];
        acc0 = fmaf(xf, av.x, acc0);
        acc1 = fmaf(xf, av.y, acc1);
        acc2 = fmaf(xf, av.z, acc2);
        acc3 = fmaf(xf, av.w, acc3);
      }
    }
  }
  cp_async_wait<0>();
  const int t = t0 + tl;
  if (t < T) {
    __nv_bfloat16* dst =
        u + (size_t)session * u_ss + (size_t)agent * u_sa + (size_t)(t + rows.u_shift) * u_st + c0 + cg * 4;
    dst[0] = __float2bfloat16_rn(acc0);
    dst[1] = __float2bfloat16_rn(acc1);
    dst[2] = __float2bfloat16_rn(acc2);
    dst[3] = __float2bfloat16_rn(acc3);
  }
}

template <int R>
void launch_r(const void* x, const void* a, const AppendRows& rows, int n, int max_len, int Dm, void* u,
              long long u_ss, long long u_sa, long long u_st, int session, cudaStream_t stream) {
  const bool fast = Dm % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 && (reinterpret_cast<uintptr_t>(a) & 15) == 0;
  if (!fast) {
    launch_generic<R>(x, a, rows, n, max_len, Dm, u, u_ss, u_sa, u_st, session, stream);
    return;
  }
  using S = FastShape<R>;
  if (ensure_dynamic_smem<append_kernel_fast<R>>(S::SMEM) != cudaSuccess) return;  // reported by the caller's check
  dim3 grid((max_len + S::TB - 1) / S::TB, n, S::NCB);
  append_kernel_fast<R><<<grid, APP_THREADS, S::SMEM, stream>>>(static_cast<const uint16_t*>(x),
                                                                 static_cast<const uint16_t*>(a), rows, Dm,
                                                                 static_cast<__nv_bfloat16*>(u), u_ss, u_sa, u_st,
                                                                 session);
}

}  // namespace

lrkv_status launch_append(const void* x, const void* a, int n_a, const int* row_begin, const int* row_end,
                          int u_shift, int Dm, int r, void* u, long long u_ss, long long u_sa, long long u_st,
                          int session, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int base = 0; base < n_a; base += kMaxAgents) {  // the ranges of up to kMaxAgents agents per launch
    AppendRows rows = {};
    rows.agent_base = base;
    rows.u_shift = u_shift;
    const int n = n_a - base < kMaxAgents ? n_a - base : kMaxAgents;
    int max_len = 0;
    for (int i = 0; i < n; ++i) {
      rows.begin[i] = row_begin[base + i];
      rows.end[i] = row_end[base + i];
      max_len = rows.end[i] - rows.begin[i] > max_len ? rows.end[i] - rows.begin[i] : max_len;
    }
    if (max_len == 0) continue;
    switch (r) {
      case 8: launch_r<8>(x, a, rows, n, max_len, Dm, u, u_ss, u_sa, u_st, session, st); break;
      case 16: launch_r<16>(x, a, rows, n, max_len, Dm, u, u_ss, u_sa, u_st, session, st); break;
      case 32: launch_r<32>(x, a, rows, n, max_len, Dm, u, u_ss, u_sa, u_st, session, st); break;
      default: return LRKV_ERR_UNSUPPORTED;
    }
    if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  }
  return LRKV_OK;
}

}  // namespace lrkv
