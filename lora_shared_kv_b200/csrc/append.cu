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

constexpr int APP_THREADS = 256;
constexpr int KC = 64;  // k-chunk staged in shared memory

__global__ void __launch_bounds__(APP_THREADS)
    append_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ a, int T, int Dm, int r,
                  __nv_bfloat16* __restrict__ u, long long u_ss, long long u_sa, long long u_st, int session,
                  int start_row) {
  extern __shared__ float sm[];
  const int ty_n = APP_THREADS / r;            // tokens per block
  float* xs = sm;                               // [ty_n][KC + 1]
  float* as = sm + ty_n * (KC + 1);             // [KC][r]
  const int tx = threadIdx.x % r;               // rank column j
  const int ty = threadIdx.x / r;               // token within the block
  const int agent = blockIdx.y;
  const int t0 = blockIdx.x * ty_n;
  const __nv_bfloat16* a_ag = a + (size_t)agent * Dm * r;
  float acc = 0.0f;
  for (int k0 = 0; k0 < Dm; k0 += KC) {
    const int kc = min(KC, Dm - k0);
    for (int i = threadIdx.x; i < ty_n * KC; i += APP_THREADS) {
      const int row = i / KC, kk = i % KC;
      const int t = t0 + row;
      xs[row * (KC + 1) + kk] = (t < T && kk < kc) ? __bfloat162float(x[(size_t)t * Dm + k0 + kk]) : 0.f;
    }
    for (int i = threadIdx.x; i < KC * r; i += APP_THREADS) {
      const int kk = i / r, j = i % r;
      as[i] = kk < kc ? __bfloat162float(a_ag[(size_t)(k0 + kk) * r + j]) : 0.f;
    }
    __syncthreads();
    if (ty < ty_n) {
      const float* xr = xs + ty * (KC + 1);
      for (int kk = 0; kk < kc; ++kk) acc = fmaf(xr[kk], as[kk * r + tx], acc);
    }
    __syncthreads();
  }
  const int t = t0 + ty;
  if (ty < ty_n && t < T) {
    u[(size_t)session * u_ss + (size_t)agent * u_sa + (size_t)(start_row + t) * u_st + tx] = __float2bfloat16_rn(acc);
  }
}

}  // namespace

lrkv_status launch_append(const void* x, const void* a, int n_a, int T, int Dm, int r, void* u, long long u_ss,
                          long long u_sa, long long u_st, int session, int start_row, void* stream) {
  if (T == 0) return LRKV_OK;
  const int ty_n = APP_THREADS / r;
  dim3 grid((T + ty_n - 1) / ty_n, n_a);
  const size_t smem = (size_t)(ty_n * (KC + 1) + KC * r) * sizeof(float);
  append_kernel<<<grid, APP_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(a), T, Dm, r,
      static_cast<__nv_bfloat16*>(u), u_ss, u_sa, u_st, session, start_row);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
