// Low-rank cache append: U_i[start + t, :] = X[t, :] A_i for new tokens.
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

// A block owns TB tokens x all r columns of one agent; a thread owns one token
// and 4 adjacent columns (4 independent fmaf chains).  X and A are staged in
// shared memory as fp32 one k-chunk at a time; the next chunk's global loads
// are issued into registers before the current chunk's FMAs, so their latency
// hides behind the arithmetic.  Each output still sums k = 0 .. Dm-1 in order.
constexpr int APP_THREADS = 128;
constexpr int X_PER_CHUNK = 2048;  // X elements staged per chunk (TB x KC)

template <int R>
struct AppShape {
  static constexpr int CG = R / 4;                    // column groups of 4
  static constexpr int TB = APP_THREADS / CG;         // tokens per block
  static constexpr int KC = X_PER_CHUNK / TB;         // k per chunk
  static constexpr int XL = X_PER_CHUNK / APP_THREADS;  // X loads per thread per chunk
  static constexpr int AL = KC * R / APP_THREADS;       // A loads per thread per chunk
  static constexpr int XS = KC + 1;                   // padded X row (conflict-free column reads)
  static_assert(APP_THREADS % KC == 0 && X_PER_CHUNK % APP_THREADS == 0 && (KC * R) % APP_THREADS == 0, "shape");
};

template <int R>
__global__ void __launch_bounds__(APP_THREADS)
    append_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ a, int T, int Dm,
                  __nv_bfloat16* __restrict__ u, long long u_ss, long long u_sa, long long u_st, int session,
                  int start_row) {
  using S = AppShape<R>;
  __shared__ float xs[S::TB * S::XS];
  __shared__ __align__(16) float as[S::KC * R];
  const int tid = threadIdx.x;
  const int tok = tid / S::CG;       // token within the block
  const int col = (tid % S::CG) * 4;  // first of this thread's 4 columns
  const int agent = blockIdx.y;
  const int t0 = blockIdx.x * S::TB;
  const uint16_t* a_ag = a + (size_t)agent * Dm * R;

  // chunk element e = tid + i * APP_THREADS sits at row e / KC, k e % KC; as
  // APP_THREADS is a multiple of KC, a thread's k is fixed and its rows step by
  // APP_THREADS / KC
  constexpr int RSTEP = APP_THREADS / S::KC;
  const int my_kk = tid % S::KC, my_row = tid / S::KC;
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
  float acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
  load_chunk(0);
  for (int k0 = 0; k0 < Dm; k0 += S::KC) {
    __syncthreads();  // the previous chunk's reads are done
#pragma unroll
    for (int i = 0; i < S::XL; ++i) xs[(my_row + i * RSTEP) * S::XS + my_kk] = __uint_as_float((uint32_t)xr[i] << 16);
#pragma unroll
    for (int i = 0; i < S::AL; ++i) as[tid + i * APP_THREADS] = __uint_as_float((uint32_t)ar[i] << 16);
    __syncthreads();
    if (k0 + S::KC < Dm) load_chunk(k0 + S::KC);
    const int kc = min(S::KC, Dm - k0);
    const float* xrow = xs + tok * S::XS;
    if (kc == S::KC) {
#pragma unroll 8
      for (int kk = 0; kk < S::KC; ++kk) {
        const float xv = xrow[kk];
        const float4 av = *reinterpret_cast<const float4*>(as + kk * R + col);
        acc0 = fmaf(xv, av.x, acc0);
        acc1 = fmaf(xv, av.y, acc1);
        acc2 = fmaf(xv, av.z, acc2);
        acc3 = fmaf(xv, av.w, acc3);
      }
    } else {
      for (int kk = 0; kk < kc; ++kk) {
        const float xv = xrow[kk];
        const float4 av = *reinterpret_cast<const float4*>(as + kk * R + col);
        acc0 = fmaf(xv, av.x, acc0);
        acc1 = fmaf(xv, av.y, acc1);
        acc2 = fmaf(xv, av.z, acc2);
        acc3 = fmaf(xv, av.w, acc3);
      }
    }
  }
  const int t = t0 + tok;
  if (t < T) {
    __nv_bfloat16* dst = u + (size_t)session * u_ss + (size_t)agent * u_sa + (size_t)(start_row + t) * u_st + col;
    dst[0] = __float2bfloat16_rn(acc0);
    dst[1] = __float2bfloat16_rn(acc1);
    dst[2] = __float2bfloat16_rn(acc2);
    dst[3] = __float2bfloat16_rn(acc3);
  }
}

template <int R>
void launch_r(const void* x, const void* a, int n_a, int T, int Dm, void* u, long long u_ss, long long u_sa,
              long long u_st, int session, int start_row, cudaStream_t stream) {
  dim3 grid((T + AppShape<R>::TB - 1) / AppShape<R>::TB, n_a);
  append_kernel<R><<<grid, APP_THREADS, 0, stream>>>(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(a),
                                                     T, Dm, static_cast<__nv_bfloat16*>(u), u_ss, u_sa, u_st,
                                                     session, start_row);
}

}  // namespace

lrkv_status launch_append(const void* x, const void* a, int n_a, int T, int Dm, int r, void* u, long long u_ss,
                          long long u_sa, long long u_st, int session, int start_row, void* stream) {
  if (T == 0) return LRKV_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (r) {
    case 8: launch_r<8>(x, a, n_a, T, Dm, u, u_ss, u_sa, u_st, session, start_row, st); break;
    case 16: launch_r<16>(x, a, n_a, T, Dm, u, u_ss, u_sa, u_st, session, start_row, st); break;
    case 32: launch_r<32>(x, a, n_a, T, Dm, u, u_ss, u_sa, u_st, session, start_row, st); break;
    default: return LRKV_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
