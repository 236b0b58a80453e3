// C ABI of liblrkv.so: argument checks, work partition, TMA descriptors,
// launches.  No allocation, no host<->device copies, no synchronisation
// (except lrkv_query_device_status, whose job it is).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include <vector>

#include "lrkv_internal.h"
#include "prefill.h"

namespace {

thread_local char g_detail[512] = "";

// Failure-detection test hook: armed by lrkv_debug_stall_next_launch, consumed
// by the next decode or prefill launch of this thread.
thread_local uint32_t g_stall_cap = 0;

// Spin cap and stall flag of a launch (disarms the hook).
void take_stall_hook(unsigned* spin_cap, int* stall) {
  *spin_cap = g_stall_cap ? g_stall_cap : lrkv::kSpinCap;
  *stall = g_stall_cap ? 1 : 0;
  g_stall_cap = 0;
}

lrkv_status fail(lrkv_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

lrkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LRKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// device facts
// ---------------------------------------------------------------------------
struct DeviceInfo {
  int sms = 0;
  int major = 0;
  int smem_optin = 0;
};

lrkv_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LRKV_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!have[dev]) {
    DeviceInfo d;
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(major)");
    if ((e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(smem)");
    cache[dev] = d;
    have[dev] = true;
  }
  *out = cache[dev];
  if (out->major != 10) return fail(LRKV_ERR_UNSUPPORTED, "needs an sm_100 GPU (found compute capability %d.x)", out->major);
  return LRKV_OK;
}

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D bf16 tensor map, dims/strides innermost first (strides in elements,
// for dims 1..3).  A dimension of extent 1 gets a packed stride.
lrkv_status make_map4(CUtensorMap* m, const void* base, const uint64_t dims[4], const int64_t strides_el[3],
                      const uint32_t box[4], CUtensorMapSwizzle swz, const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(LRKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t gdim[4];
  cuuint64_t gstr[3];
  uint64_t packed = dims[0] * 2;
  for (int i = 0; i < 4; ++i) gdim[i] = dims[i];
  for (int i = 0; i < 3; ++i) {
    uint64_t s = strides_el[i] > 0 ? (uint64_t)strides_el[i] * 2 : 0;
    if (dims[i + 1] == 1 || s == 0) s = packed < 16 ? 16 : (packed + 15) / 16 * 16;
    if (s % 16 != 0) return fail(LRKV_ERR_MISALIGNED, "%s: stride %d (%llu bytes) is not a multiple of 16 bytes", what, i + 1, (unsigned long long)s);
    gstr[i] = s;
    packed = s * dims[i + 1];
  }
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim, gstr, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LRKV_ERR_INVALID_ARGUMENT, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
  return LRKV_OK;
}

// ---------------------------------------------------------------------------
// shared checks
// ---------------------------------------------------------------------------
lrkv_status check_problem(const lrkv_problem* p) {
  if (!p) return fail(LRKV_ERR_INVALID_ARGUMENT, "problem is NULL");
  if (p->num_sessions < 1 || p->num_agents < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "sessions, agents and heads must be >= 1");
  if (p->num_q_heads % p->num_kv_heads != 0)
    return fail(LRKV_ERR_UNSUPPORTED, "num_q_heads (%d) must be a multiple of num_kv_heads (%d)", p->num_q_heads, p->num_kv_heads);
  if (p->head_dim != 64 && p->head_dim != 128) return fail(LRKV_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", p->head_dim);
  if (p->rank != 8 && p->rank != 16 && p->rank != 32) return fail(LRKV_ERR_UNSUPPORTED, "rank %d (supported: 8, 16, 32)", p->rank);
  if (p->mode != LRKV_BASE_SHARED && p->mode != LRKV_BASE_LR_SHARED) return fail(LRKV_ERR_INVALID_ARGUMENT, "mode %d", p->mode);
  if (p->num_agents > lrkv::kMaxAgents) return fail(LRKV_ERR_UNSUPPORTED, "at most %d agents per call", lrkv::kMaxAgents);
  if (!(p->softmax_scale >= 0.f) || isinf(p->softmax_scale)) return fail(LRKV_ERR_INVALID_ARGUMENT, "softmax_scale must be finite and >= 0");
  return LRKV_OK;
}

float scale_of(const lrkv_problem* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf((float)p->head_dim);
}

lrkv_status check_kv(const lrkv_kv_view* kv, const lrkv_problem* p) {
  if (!kv || !kv->k || !kv->v) return fail(LRKV_ERR_INVALID_ARGUMENT, "kv view or its k/v pointer is NULL");
  if (!aligned16(kv->k) || !aligned16(kv->v)) return fail(LRKV_ERR_MISALIGNED, "k and v must be 16-byte aligned");
  if (kv->stride_token < p->head_dim || kv->stride_head < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "kv strides too small");
  if (kv->stride_token % 8 || kv->stride_head % 8) return fail(LRKV_ERR_MISALIGNED, "kv token/head strides must be multiples of 8 elements");
  if (kv->page_table) {
    if (kv->page_size != lrkv::kKeysPerTile) return fail(LRKV_ERR_UNSUPPORTED, "page_size %d (supported: 64)", kv->page_size);
    if (kv->num_pages < 1 || kv->stride_page < 1 || kv->stride_page % 8) return fail(LRKV_ERR_INVALID_ARGUMENT, "paged view needs num_pages >= 1 and a stride_page that is a positive multiple of 8");
    if (kv->page_table_stride < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "page_table_stride must be >= 1");
  } else {
    if (p->num_sessions > 1 && (kv->stride_session < 1 || kv->stride_session % 8)) return fail(LRKV_ERR_MISALIGNED, "kv session stride must be a positive multiple of 8 elements");
  }
  return LRKV_OK;
}

lrkv_status check_u(const lrkv_u_view* u, const lrkv_problem* p, int rows_needed) {
  if (!u || !u->u) return fail(LRKV_ERR_INVALID_ARGUMENT, "u view or its pointer is NULL");
  if (!aligned16(u->u)) return fail(LRKV_ERR_MISALIGNED, "u must be 16-byte aligned");
  if (u->stride_token < p->rank || u->stride_token % 8) return fail(LRKV_ERR_MISALIGNED, "u stride_token must be >= rank and a multiple of 8");
  const int slots = p->mode == LRKV_BASE_SHARED ? p->num_agents : 1;
  if (slots > 1 && (u->stride_agent < 1 || u->stride_agent % 8)) return fail(LRKV_ERR_MISALIGNED, "u stride_agent must be a positive multiple of 8");
  if (p->num_sessions > 1 && (u->stride_session < 1 || u->stride_session % 8)) return fail(LRKV_ERR_MISALIGNED, "u stride_session must be a positive multiple of 8");
  if (u->num_rows < rows_needed) return fail(LRKV_ERR_INVALID_ARGUMENT, "u num_rows %d < %d rows needed", u->num_rows, rows_needed);
  return LRKV_OK;
}

// ---------------------------------------------------------------------------
// decode plan
// ---------------------------------------------------------------------------
struct DecodePlan {
  int G, R, n_rg, rows_per_group, NT, n_u_slots, nt, items, ctas, max_segs, groups, stages, smem;
  long long W;
  size_t tickets_off, partials_off, bytes;
};

// Work partition of one decode launch over `hkv` KV heads (all of the
// problem's, or a shard of them).
lrkv_status plan_decode(const lrkv_problem* p, int hkv, int max_seq_len, const DeviceInfo& dev, DecodePlan* pl) {
  lrkv_status s = check_problem(p);
  if (s != LRKV_OK) return s;
  if (hkv < 1 || hkv > p->num_kv_heads) return fail(LRKV_ERR_INVALID_ARGUMENT, "KV-head count %d of %d", hkv, p->num_kv_heads);
  if (max_seq_len < 0) return fail(LRKV_ERR_INVALID_ARGUMENT, "max_seq_len must be >= 0");
  pl->G = p->num_q_heads / p->num_kv_heads;
  pl->R = p->num_agents * pl->G;
  pl->n_rg = (pl->R + lrkv::kMaxRowsPerItem - 1) / lrkv::kMaxRowsPerItem;
  pl->rows_per_group = (pl->R + pl->n_rg - 1) / pl->n_rg;
  pl->NT = (pl->rows_per_group + 7) / 8;
  int max_ag = 0;
  for (int rg = 0; rg < pl->n_rg; ++rg) {
    const int lo = rg * pl->rows_per_group;
    const int hi = lo + pl->rows_per_group < pl->R ? lo + pl->rows_per_group : pl->R;
    if (hi <= lo) continue;
    const int n = (hi - 1) / pl->G - lo / pl->G + 1;
    max_ag = n > max_ag ? n : max_ag;
  }
  pl->n_u_slots = p->mode == LRKV_BASE_SHARED ? max_ag : 1;
  pl->nt = max_seq_len > 0 ? (max_seq_len + lrkv::kKeysPerTile - 1) / lrkv::kKeysPerTile : 1;
  pl->items = p->num_sessions * hkv * pl->n_rg;
  pl->W = (long long)pl->items * pl->nt;
  const int sms = dev.sms > 0 ? dev.sms : 148;
  pl->ctas = (int)(pl->W < sms ? pl->W : sms);
  // Whole items, one per CTA, when there are no more items than SMs and the even
  // split would take fewer than kWholeItemSlackTiles tiles off a CTA: an item
  // split over CTAs pays for publishing its partial records, a ticket and their
  // merge at the end of the launch.  (Measured on Qwen3 shapes with 128 items
  // of 16 / 32 / 64 tiles: 0.633 -> 0.510, 0.869 -> 0.779 and 1.378 -> 1.332 ms
  // per 28 layers; a fit gives about 5.4 us per launch for the split against
  // 0.44 us per extra tile.)
  if (pl->items <= sms && pl->nt <= (int)((pl->W + pl->ctas - 1) / pl->ctas) + lrkv::kWholeItemSlackTiles)
    pl->ctas = pl->items;
  int ms = 1;
  for (int it = 0; it < pl->items; ++it) {
    const long long cf = lrkv::owner_cta((long long)it * pl->nt, pl->W, pl->ctas);
    const long long cl = lrkv::owner_cta((long long)(it + 1) * pl->nt - 1, pl->W, pl->ctas);
    const int n = (int)(cl - cf + 1);
    ms = n > ms ? n : ms;
  }
  pl->max_segs = ms;
  pl->groups = lrkv::decode_groups(pl->NT, ms > 1);
  // shared memory: as many stages as fit (2..8)
  const int optin = dev.smem_optin > 0 ? dev.smem_optin : 232448;
  int stages = 8;
  for (; stages >= 2; --stages) {
    lrkv::DecodeSmem lay = lrkv::decode_smem_plan(p->head_dim, pl->NT, p->rank, pl->n_u_slots, stages);
    if (lay.total + 1024 <= optin) break;
  }
  if (stages < 2) return fail(LRKV_ERR_UNSUPPORTED, "decode tiles do not fit in shared memory");
  pl->stages = stages;
  pl->smem = lrkv::decode_smem_plan(p->head_dim, pl->NT, p->rank, pl->n_u_slots, stages).total + 1024;
  pl->tickets_off = lrkv::kWsHeaderBytes;
  pl->partials_off = pl->tickets_off + ((size_t)pl->items * 4 + 255) / 256 * 256;
  const size_t rec = lrkv::decode_record_floats(pl->NT, p->head_dim, p->rank) * 4;
  pl->bytes = pl->partials_off + (pl->max_segs > 1 ? (size_t)pl->items * pl->max_segs * rec : 0);
  return LRKV_OK;
}

}  // namespace

extern "C" {

const char* lrkv_status_string(lrkv_status s) {
  switch (s) {
    case LRKV_OK: return "ok";
    case LRKV_ERR_INVALID_ARGUMENT: return "invalid argument";
    case LRKV_ERR_UNSUPPORTED: return "unsupported";
    case LRKV_ERR_MISALIGNED: return "misaligned";
    case LRKV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case LRKV_ERR_CUDA: return "CUDA error";
    case LRKV_ERR_DEVICE_FAULT: return "device-side check failed";
    case LRKV_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* lrkv_last_error_detail(void) { return g_detail; }

lrkv_status lrkv_debug_stall_next_launch(uint32_t spin_cap) {
  g_stall_cap = spin_cap;
  return LRKV_OK;
}

int32_t lrkv_version(void) { return 100; }

lrkv_status lrkv_value_projection(const lrkv_problem* p, const void* x, int32_t T, int32_t Dm, const void* w,
                                  const lrkv_kv_view* kv, int32_t kv_rows, const lrkv_u_view* u_dst,
                                  int32_t session, int32_t start_row, void* workspace, size_t workspace_bytes,
                                  lrkv_stream_t stream) {
  lrkv_status s = check_problem(p);
  if (s != LRKV_OK) return s;
  if (!x || !w || !kv || !kv->v || !u_dst || !u_dst->u || !workspace)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "x, w, kv->v, u_dst->u and workspace must not be NULL");
  if (T < 0 || Dm < 1 || session < 0 || start_row < 0)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "need T >= 0, Dm >= 1, session >= 0, start_row >= 0");
  if (!kv->page_table && session >= p->num_sessions)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "session %d >= num_sessions %d", session, p->num_sessions);
  if (Dm % 8) return fail(LRKV_ERR_MISALIGNED, "Dm must be a multiple of 8 (16-byte rows of x)");
  if (!aligned16(x) || !aligned16(w) || !aligned16(kv->v) || !aligned16(u_dst->u) || !aligned16(workspace))
    return fail(LRKV_ERR_MISALIGNED, "x, w, kv->v, u and workspace must be 16-byte aligned");
  if (workspace_bytes < (size_t)lrkv::kWsHeaderBytes)
    return fail(LRKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %d bytes", workspace_bytes, lrkv::kWsHeaderBytes);
  if ((kv->stride_token % 8) || (kv->stride_head % 8) || (!kv->page_table && (kv->stride_session % 8)) ||
      (kv->page_table && (kv->stride_page % 8)))
    return fail(LRKV_ERR_MISALIGNED, "kv strides must be multiples of 8 elements");
  const int n_u = p->mode == LRKV_BASE_SHARED ? p->num_agents : 1;
  if ((s = check_u(u_dst, p, start_row + T)) != LRKV_OK) return s;
  if (kv->page_table) {
    if (kv->page_size < 1 || kv->num_pages < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "paged view needs page_size and num_pages");
    if ((long long)(start_row + T + kv->page_size - 1) / kv->page_size > kv->page_table_stride)
      return fail(LRKV_ERR_INVALID_ARGUMENT, "rows past the session's page-table row");
  } else if (start_row + T > kv_rows) {
    return fail(LRKV_ERR_INVALID_ARGUMENT, "rows [%d, %d) exceed the value cache's %d rows", start_row, start_row + T, kv_rows);
  }
  if (T == 0) return LRKV_OK;
  DeviceInfo dev;
  if ((s = device_info(&dev)) != LRKV_OK) return s;
  const int ncols = p->num_kv_heads * p->head_dim + n_u * p->rank;
  alignas(64) CUtensorMap maps[2];
  {  // X [T, Dm]: box 64 k x 128 tokens
    const uint64_t dims[4] = {(uint64_t)Dm, (uint64_t)T, 1, 1};
    const int64_t str[3] = {Dm, 0, 0};
    const uint32_t box[4] = {64, 128, 1, 1};
    if ((s = make_map4(&maps[0], x, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, "X")) != LRKV_OK) return s;
  }
  {  // W [Dm, ncols]: box 64 columns x 64 k
    const uint64_t dims[4] = {(uint64_t)ncols, (uint64_t)Dm, 1, 1};
    const int64_t str[3] = {ncols, 0, 0};
    const uint32_t box[4] = {64, 64, 1, 1};
    if ((s = make_map4(&maps[1], w, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, "W")) != LRKV_OK) return s;
  }
  lrkv::VprojParams vp = {};
  vp.T = T;
  vp.Dm = Dm;
  vp.Hkv = p->num_kv_heads;
  vp.d = p->head_dim;
  vp.n_u = n_u;
  vp.r = p->rank;
  vp.ncols = ncols;
  vp.start_row = start_row;
  vp.session = session;
  vp.v = static_cast<uint16_t*>(const_cast<void*>(kv->v));
  vp.v_ss = kv->stride_session;
  vp.v_sh = kv->stride_head;
  vp.v_st = kv->stride_token;
  vp.v_sp = kv->stride_page;
  vp.page_table = kv->page_table;
  vp.pt_stride = kv->page_table_stride;
  vp.page_size = kv->page_size;
  vp.num_pages = kv->num_pages;
  vp.u = static_cast<uint16_t*>(u_dst->u);
  vp.u_ss = u_dst->stride_session;
  vp.u_sa = u_dst->stride_agent;
  vp.u_st = u_dst->stride_token;
  vp.flags = static_cast<unsigned*>(workspace);
  s = lrkv::launch_vproj(vp, &maps[0], &maps[1], dev.sms, stream);
  if (s != LRKV_OK) return fail(s, "value projection launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  return LRKV_OK;
}

lrkv_status lrkv_workspace_reset(void* workspace, size_t workspace_bytes, lrkv_stream_t stream) {
  if (!workspace) return fail(LRKV_ERR_INVALID_ARGUMENT, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return LRKV_OK;
}

}  // extern "C"

namespace {

// Read (and optionally clear) the flag word at the start of a workspace on
// `stream`, then turn its bits into a status.
lrkv_status read_device_flags(const void* workspace, int32_t clear, uint32_t* flags_out, lrkv_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t flags = 0;
  cudaError_t e = cudaMemcpyAsync(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace flags");
  if (clear && flags) {
    e = cudaMemsetAsync(const_cast<void*>(workspace), 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace flags");
  }
  if (flags_out) *flags_out = flags;
  if (flags & LRKV_DEVFLAG_TIMEOUT) return fail(LRKV_ERR_TIMEOUT, "a bounded wait inside a kernel gave up (flags 0x%x)", flags);
  if (flags) return fail(LRKV_ERR_DEVICE_FAULT, "device-side checks flagged bad data (flags 0x%x: %s%s%s)", flags,
                         (flags & LRKV_DEVFLAG_SEQLEN) ? "seq_len " : "", (flags & LRKV_DEVFLAG_OFFSET) ? "offset " : "",
                         (flags & LRKV_DEVFLAG_PAGE) ? "page-id" : "");
  return LRKV_OK;
}

}  // namespace

extern "C" {

lrkv_status lrkv_query_device_status(const void* workspace, int32_t clear, uint32_t* flags_out,
                                     lrkv_stream_t stream) {
  if (!workspace) return fail(LRKV_ERR_INVALID_ARGUMENT, "workspace is NULL");
  return read_device_flags(workspace, clear, flags_out, stream);
}

lrkv_status lrkv_append_lr_cache(const void* x, const void* a, int32_t n_a, int32_t T, int32_t Dm, int32_t r,
                                 const lrkv_u_view* u_dst, int32_t session, int32_t start_row,
                                 lrkv_stream_t stream) {
  if (!x || !a || !u_dst || !u_dst->u) return fail(LRKV_ERR_INVALID_ARGUMENT, "x, a and u_dst->u must not be NULL");
  if (T < 0 || Dm < 1 || n_a < 1 || session < 0 || start_row < 0)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "need T >= 0, Dm >= 1, n_a >= 1, session >= 0, start_row >= 0");
  if (r != 8 && r != 16 && r != 32) return fail(LRKV_ERR_UNSUPPORTED, "rank %d (supported: 8, 16, 32)", r);
  if ((long long)start_row + T > u_dst->num_rows)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "rows [%d, %lld) exceed the U capacity %d", start_row, (long long)start_row + T, u_dst->num_rows);
  if (u_dst->stride_token < r) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_token < rank");
  if (n_a > 1 && u_dst->stride_agent < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_agent must be >= 1 when n_a > 1");
  if (session > 0 && u_dst->stride_session < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_session must be >= 1");
  if (T == 0) return LRKV_OK;
  DeviceInfo dev;
  lrkv_status s = device_info(&dev);
  if (s != LRKV_OK) return s;
  std::vector<int> begin(n_a, 0), end(n_a, T);
  s = lrkv::launch_append(x, a, n_a, begin.data(), end.data(), start_row, Dm, r, u_dst->u, u_dst->stride_session,
                          u_dst->stride_agent, u_dst->stride_token, session, stream);
  if (s != LRKV_OK) return fail(s, "append launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  return LRKV_OK;
}

lrkv_status lrkv_append_lr_cache_ranges(const void* x, int32_t x_rows, const void* a, int32_t n_a, int32_t Dm,
                                        int32_t r, const int32_t* row_begin, const int32_t* row_end,
                                        const lrkv_u_view* u_dst, int32_t session, lrkv_stream_t stream) {
  if (!x || !a || !u_dst || !u_dst->u || !row_begin || !row_end)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "x, a, row_begin, row_end and u_dst->u must not be NULL");
  if (x_rows < 0 || Dm < 1 || n_a < 1 || session < 0)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "need x_rows >= 0, Dm >= 1, n_a >= 1, session >= 0");
  if (r != 8 && r != 16 && r != 32) return fail(LRKV_ERR_UNSUPPORTED, "rank %d (supported: 8, 16, 32)", r);
  if (u_dst->stride_token < r) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_token < rank");
  if (n_a > 1 && u_dst->stride_agent < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_agent must be >= 1 when n_a > 1");
  if (session > 0 && u_dst->stride_session < 1) return fail(LRKV_ERR_INVALID_ARGUMENT, "u stride_session must be >= 1");
  bool any = false;
  for (int i = 0; i < n_a; ++i) {
    if (row_begin[i] < 0 || row_begin[i] > row_end[i])
      return fail(LRKV_ERR_INVALID_ARGUMENT, "agent %d: need 0 <= row_begin <= row_end (got %d, %d)", i, row_begin[i], row_end[i]);
    if (row_end[i] > x_rows || row_end[i] > u_dst->num_rows)
      return fail(LRKV_ERR_INVALID_ARGUMENT, "agent %d: row_end %d exceeds x_rows %d or the U capacity %d", i, row_end[i], x_rows, u_dst->num_rows);
    any = any || row_end[i] > row_begin[i];
  }
  if (!any) return LRKV_OK;
  DeviceInfo dev;
  lrkv_status s = device_info(&dev);
  if (s != LRKV_OK) return s;
  s = lrkv::launch_append(x, a, n_a, row_begin, row_end, 0, Dm, r, u_dst->u, u_dst->stride_session,
                          u_dst->stride_agent, u_dst->stride_token, session, stream);
  if (s != LRKV_OK) return fail(s, "append launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  return LRKV_OK;
}

size_t lrkv_decode_workspace_bytes(const lrkv_problem* p, int32_t max_seq_len) {
  DeviceInfo dev;
  if (device_info(&dev) != LRKV_OK) {
    dev.sms = 148;
    dev.smem_optin = 232448;
  }
  DecodePlan pl;
  if (plan_decode(p, p ? p->num_kv_heads : 0, max_seq_len, dev, &pl) != LRKV_OK) return 0;
  return pl.bytes;
}

}  // extern "C"

namespace {

// Decode over KV heads [g_begin, g_begin + g_count) of the problem: the K/V
// view holds those heads only (its head 0 is head g_begin); q, out and B are
// the whole problem's, and only the query heads of these KV heads are written.
lrkv_status decode_heads(const lrkv_problem* p, int g_begin, int g_count, const void* q, const lrkv_kv_view* kv,
                         const int32_t* seq_lens, int32_t max_seq_len, const lrkv_u_view* u, const void* b,
                         const int32_t* alora_offsets, void* out, int32_t out_dtype, void* workspace,
                         size_t workspace_bytes, lrkv_stream_t stream) {
  lrkv_status s = check_problem(p);
  if (s != LRKV_OK) return s;
  if (g_begin < 0 || g_count < 1 || (long long)g_begin + g_count > p->num_kv_heads)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "KV heads [%d, %d + %d) outside [0, %d)", g_begin, g_begin, g_count, p->num_kv_heads);
  if (!q || !seq_lens || !b || !out || !workspace) return fail(LRKV_ERR_INVALID_ARGUMENT, "q, seq_lens, b, out and workspace must not be NULL");
  if (!aligned16(q) || !aligned16(b) || !aligned16(out) || !aligned16(workspace)) return fail(LRKV_ERR_MISALIGNED, "q, b, out and workspace must be 16-byte aligned");
  if (out_dtype != LRKV_BF16 && out_dtype != LRKV_F32) return fail(LRKV_ERR_INVALID_ARGUMENT, "out_dtype %d", out_dtype);
  if ((s = check_kv(kv, p)) != LRKV_OK) return s;
  if ((s = check_u(u, p, max_seq_len)) != LRKV_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(&dev)) != LRKV_OK) return s;
  DecodePlan pl;
  if ((s = plan_decode(p, g_count, max_seq_len, dev, &pl)) != LRKV_OK) return s;
  if (workspace_bytes < pl.bytes) return fail(LRKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, pl.bytes);

  const int D = p->head_dim, RK = p->rank;
  const int Lmap = max_seq_len > 0 ? max_seq_len : 1;
  alignas(64) CUtensorMap tmK, tmV, tmU;
  const uint32_t kbox[4] = {64, (uint32_t)lrkv::kKeysPerTile, 1, 1};
  if (kv->page_table) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)kv->page_size, (uint64_t)g_count, (uint64_t)kv->num_pages};
    const int64_t str[3] = {kv->stride_token, kv->stride_head, kv->stride_page};
    if ((s = make_map4(&tmK, kv->k, dims, str, kbox, CU_TENSOR_MAP_SWIZZLE_128B, "K pages")) != LRKV_OK) return s;
    if ((s = make_map4(&tmV, kv->v, dims, str, kbox, CU_TENSOR_MAP_SWIZZLE_128B, "V pages")) != LRKV_OK) return s;
  } else {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Lmap, (uint64_t)g_count, (uint64_t)p->num_sessions};
    const int64_t str[3] = {kv->stride_token, kv->stride_head, kv->stride_session};
    if ((s = make_map4(&tmK, kv->k, dims, str, kbox, CU_TENSOR_MAP_SWIZZLE_128B, "K")) != LRKV_OK) return s;
    if ((s = make_map4(&tmV, kv->v, dims, str, kbox, CU_TENSOR_MAP_SWIZZLE_128B, "V")) != LRKV_OK) return s;
  }
  {
    const int slots = p->mode == LRKV_BASE_SHARED ? p->num_agents : 1;
    const uint64_t dims[4] = {(uint64_t)RK, (uint64_t)u->num_rows, (uint64_t)slots, (uint64_t)p->num_sessions};
    const int64_t str[3] = {u->stride_token, u->stride_agent, u->stride_session};
    const uint32_t ubox[4] = {(uint32_t)RK, (uint32_t)lrkv::kKeysPerTile, 1, 1};
    if ((s = make_map4(&tmU, u->u, dims, str, ubox, CU_TENSOR_MAP_SWIZZLE_NONE, "U")) != LRKV_OK) return s;
  }

  lrkv::DecodeParams dp = {};
  dp.q = q;
  dp.b = b;
  dp.seq_lens = seq_lens;
  dp.offsets = alora_offsets;
  dp.page_table = kv->page_table;
  dp.pt_stride = kv->page_table_stride;
  dp.out = out;
  dp.out_f32 = out_dtype == LRKV_F32;
  dp.S = p->num_sessions;
  dp.N = p->num_agents;
  dp.Hq = p->num_q_heads;
  dp.Hkv = g_count;
  dp.g_base = g_begin;
  dp.Hkv_total = p->num_kv_heads;
  dp.G = pl.G;
  dp.rows_total = pl.R;
  dp.rows_per_group = pl.rows_per_group;
  dp.n_rg = pl.n_rg;
  dp.n_u_slots = pl.n_u_slots;
  dp.mode = p->mode;
  dp.max_seq_len = max_seq_len;
  dp.u_rows = u->num_rows;
  dp.num_pages = kv->page_table ? kv->num_pages : 0;
  dp.paged = kv->page_table != nullptr;
  dp.nt = pl.nt;
  {
    // Visiting order of an item's tiles.  Tiles past an agent's offset carry
    // its U tile and low-rank MMAs; when those are a sizeable share of a tile's
    // work (BaseShared with n_agents * r >= d / 4, i.e. U bytes >= an eighth of
    // the K+V bytes) they must be spread evenly over the CTAs sharing an item,
    // so runs of tiles are visited in a low-discrepancy order (stride coprime
    // to the run count, near 0.618 of it).  Otherwise plain ascending order
    // streams HBM best (stride 1).  (Measured on the Qwen2.5 case, 3 agents at
    // r = 16, d = 128: 1.773 ms per step in order, 1.748 balanced; a probe of
    // one launch showed the CTAs' loop end times correlated with their U tile
    // counts, 0.6, in order.)
    const int runs = pl.nt / lrkv::kTileRun;
    const bool balance = p->mode == LRKV_BASE_SHARED && pl.n_u_slots * p->rank * 4 >= p->head_dim;
    int stride = 1;
    if (balance && runs > 1) {
      stride = (int)(0.618 * runs) | 1;
      auto gcd = [](long long x, long long y) { while (y) { long long t = x % y; x = y; y = t; } return x; };
      while (gcd(stride, runs) != 1) stride += 2;
      if (stride % runs == 0) stride = 1;
    }
    dp.tile_stride = stride;
  }
  dp.items = pl.items;
  dp.W = pl.W;
  dp.max_segs = pl.max_segs;
  dp.stages = pl.stages;
  dp.scale_log2 = scale_of(p) * 1.4426950408889634f;
  char* ws = static_cast<char*>(workspace);
  dp.flags = reinterpret_cast<unsigned*>(ws);
  dp.tickets = reinterpret_cast<int*>(ws + pl.tickets_off);
  dp.partials = reinterpret_cast<float*>(ws + pl.partials_off);
  take_stall_hook(&dp.spin_cap, &dp.stall);
  s = lrkv::launch_decode(dp, D, pl.NT, RK, pl.groups, &tmK, &tmV, &tmU, pl.smem, pl.ctas, stream);
  if (s != LRKV_OK) return fail(s, "decode launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  return LRKV_OK;
}

}  // namespace

extern "C" {

lrkv_status lrkv_attn_decode(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv, const int32_t* seq_lens,
                             int32_t max_seq_len, const lrkv_u_view* u, const void* b,
                             const int32_t* alora_offsets, void* out, int32_t out_dtype, void* workspace,
                             size_t workspace_bytes, lrkv_stream_t stream) {
  return decode_heads(p, 0, p ? p->num_kv_heads : 0, q, kv, seq_lens, max_seq_len, u, b, alora_offsets, out,
                      out_dtype, workspace, workspace_bytes, stream);
}

size_t lrkv_decode_kv_heads_workspace_bytes(const lrkv_problem* p, int32_t kv_head_count, int32_t max_seq_len) {
  DeviceInfo dev;
  if (device_info(&dev) != LRKV_OK) {
    dev.sms = 148;
    dev.smem_optin = 232448;
  }
  DecodePlan pl;
  if (plan_decode(p, kv_head_count, max_seq_len, dev, &pl) != LRKV_OK) return 0;
  return pl.bytes;
}

lrkv_status lrkv_attn_decode_kv_heads(const lrkv_problem* p, int32_t kv_head_begin, int32_t kv_head_count,
                                      const void* q, const lrkv_kv_view* kv, const int32_t* seq_lens,
                                      int32_t max_seq_len, const lrkv_u_view* u, const void* b,
                                      const int32_t* alora_offsets, void* out, int32_t out_dtype, void* workspace,
                                      size_t workspace_bytes, lrkv_stream_t stream) {
  return decode_heads(p, kv_head_begin, kv_head_count, q, kv, seq_lens, max_seq_len, u, b, alora_offsets, out,
                      out_dtype, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Decode with library-owned scratch: for callers that may not allocate device
// memory.  The scratch is one file-scope device array (every GPU that loads the
// library holds it until the process exits).
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)8 << 20;  // LRKV_STATIC_SCRATCH_BYTES in lrkv.h
static_assert(kStaticScratchBytes == LRKV_STATIC_SCRATCH_BYTES, "header and library disagree on the scratch size");

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device, looked up once per
// device (the host-side name of the array is not a device address).
lrkv_status static_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LRKV_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || ptr == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    addr[dev] = ptr;
  }
  *out = addr[dev];
  return LRKV_OK;
}

}  // namespace

extern "C" {

lrkv_status lrkv_attn_decode_static_scratch(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv,
                                            const int32_t* seq_lens, int32_t max_seq_len, const lrkv_u_view* u,
                                            const void* b, const int32_t* alora_offsets, void* out,
                                            int32_t out_dtype, lrkv_stream_t stream) {
  lrkv_status s = check_problem(p);
  if (s != LRKV_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(&dev)) != LRKV_OK) return s;
  DecodePlan pl;
  if ((s = plan_decode(p, p->num_kv_heads, max_seq_len, dev, &pl)) != LRKV_OK) return s;
  if (pl.bytes > kStaticScratchBytes)
    return fail(LRKV_ERR_WORKSPACE_TOO_SMALL,
                "this shape needs %zu bytes of decode scratch; the library's fixed scratch holds %zu "
                "(use lrkv_attn_decode with a caller-owned workspace)", pl.bytes, kStaticScratchBytes);
  void* scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != LRKV_OK) return s;
  // flags and per-item tickets must start at zero; the partial records need no clearing
  cudaError_t e = cudaMemsetAsync(scratch, 0, pl.partials_off, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(decode scratch header)");
  return lrkv_attn_decode(p, q, kv, seq_lens, max_seq_len, u, b, alora_offsets, out, out_dtype, scratch,
                          kStaticScratchBytes, stream);
}

// The flags of the most recent static-scratch call (every call clears them first).
lrkv_status lrkv_query_static_scratch_status(int32_t clear, uint32_t* flags_out, lrkv_stream_t stream) {
  void* scratch = nullptr;
  lrkv_status s = static_scratch_address(&scratch);
  if (s != LRKV_OK) return s;
  return read_device_flags(scratch, clear, flags_out, stream);
}

}  // extern "C"

namespace {

// Shape rules of the prefill chunk beyond check_problem: a 128-row tile holds
// floor(128 / G) tokens x G query heads, so G may be at most 128.
lrkv_status check_prefill_shape(const lrkv_problem* p, int32_t ctx_len, int32_t T) {
  lrkv_status s = check_problem(p);
  if (s != LRKV_OK) return s;
  if (ctx_len < 0 || T < 0) return fail(LRKV_ERR_INVALID_ARGUMENT, "need ctx_len >= 0 and T >= 0");
  if ((long long)ctx_len + T > 0x7fffffffLL) return fail(LRKV_ERR_INVALID_ARGUMENT, "ctx_len + T overflows");
  const int G = p->num_q_heads / p->num_kv_heads;
  if (G > 128) return fail(LRKV_ERR_UNSUPPORTED, "prefill needs Hq / Hkv <= 128 (got %d)", G);
  return LRKV_OK;
}

// Rank of the kernel instance that serves rank r: rank 8 runs in the rank-16
// instance, whose U and B tiles are 16 wide; the tensor maps of U and B keep
// their true rank, so the Tensor Memory Accelerator fills ranks 8..15 with zeros.
int prefill_kernel_rank(int r) { return r == 8 ? 16 : r; }

}  // namespace

extern "C" {

size_t lrkv_prefill_workspace_bytes(const lrkv_problem* p, int32_t ctx_len, int32_t T) {
  if (check_prefill_shape(p, ctx_len, T) != LRKV_OK) return 0;
  if (T == 0) return lrkv::kWsHeaderBytes;
  DeviceInfo dev;
  if (device_info(&dev) != LRKV_OK) dev.sms = 148;
  const int G = p->num_q_heads / p->num_kv_heads;
  return lrkv::plan_prefill(T, ctx_len, G, p->num_kv_heads, p->num_agents, p->head_dim, dev.sms).bytes;
}

lrkv_status lrkv_attn_prefill_chunk(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv, int32_t session,
                                    int32_t ctx_len, int32_t T, const lrkv_u_view* u, const void* b,
                                    const int32_t* alora_offsets, void* out, int32_t out_dtype, void* workspace,
                                    size_t workspace_bytes, lrkv_stream_t stream) {
  lrkv_status s = check_prefill_shape(p, ctx_len, T);
  if (s != LRKV_OK) return s;
  if (!q || !b || !out || !workspace) return fail(LRKV_ERR_INVALID_ARGUMENT, "q, b, out and workspace must not be NULL");
  if (!aligned16(q) || !aligned16(b) || !aligned16(out) || !aligned16(workspace))
    return fail(LRKV_ERR_MISALIGNED, "q, b, out and workspace must be 16-byte aligned");
  if (out_dtype != LRKV_BF16 && out_dtype != LRKV_F32) return fail(LRKV_ERR_INVALID_ARGUMENT, "out_dtype %d", out_dtype);
  if (session < 0 || session >= p->num_sessions)
    return fail(LRKV_ERR_INVALID_ARGUMENT, "need 0 <= session < num_sessions (got %d of %d)", session, p->num_sessions);
  const int G = p->num_q_heads / p->num_kv_heads;
  const long long Ltot = (long long)ctx_len + T;
  if ((s = check_kv(kv, p)) != LRKV_OK) return s;
  if ((s = check_u(u, p, (int)Ltot)) != LRKV_OK) return s;
  if (workspace_bytes < (size_t)lrkv::kWsHeaderBytes) return fail(LRKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %d bytes", workspace_bytes, lrkv::kWsHeaderBytes);
  if (T == 0) return LRKV_OK;
  DeviceInfo dev;
  if ((s = device_info(&dev)) != LRKV_OK) return s;
  // RK: the width of the U and B tiles (the kernel instance); p->rank: the caches' true rank
  const int D = p->head_dim, RK = prefill_kernel_rank(p->rank);
  if (lrkv::prefill_smem_bytes(D, RK) > dev.smem_optin) return fail(LRKV_ERR_UNSUPPORTED, "prefill tiles do not fit in shared memory");

  alignas(64) CUtensorMap maps[4];
  // V and U blocks sit side by side in shared memory as one [keys, d + r]
  // operand of RK-element swizzle atoms, so that P [V | U | 1] is one MMA per k-step
  const CUtensorMapSwizzle vu_swizzle = RK == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (kv->page_table) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)kv->page_size, (uint64_t)p->num_kv_heads, (uint64_t)kv->num_pages};
    const int64_t str[3] = {kv->stride_token, kv->stride_head, kv->stride_page};
    const uint32_t box[4] = {64, 64, 1, 1};
    const uint32_t vbox[4] = {(uint32_t)RK, 64, 1, 1};  // V in the same RK-wide swizzle atoms as U
    if ((s = make_map4(&maps[0], kv->k, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, "K pages")) != LRKV_OK) return s;
    if ((s = make_map4(&maps[1], kv->v, dims, str, vbox, vu_swizzle, "V pages")) != LRKV_OK) return s;
  } else {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Ltot, (uint64_t)p->num_kv_heads, (uint64_t)p->num_sessions};
    const int64_t str[3] = {kv->stride_token, kv->stride_head, kv->stride_session};
    const uint32_t box[4] = {64, 128, 1, 1};
    const uint32_t vbox[4] = {(uint32_t)RK, 128, 1, 1};
    if ((s = make_map4(&maps[0], kv->k, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, "K")) != LRKV_OK) return s;
    if ((s = make_map4(&maps[1], kv->v, dims, str, vbox, vu_swizzle, "V")) != LRKV_OK) return s;
  }
  {
    // the box is RK wide; ranks past p->rank lie outside the map and arrive as zeros
    const int slots = p->mode == LRKV_BASE_SHARED ? p->num_agents : 1;
    const uint64_t dims[4] = {(uint64_t)p->rank, (uint64_t)Ltot, (uint64_t)slots, (uint64_t)p->num_sessions};
    const int64_t str[3] = {u->stride_token, u->stride_agent, u->stride_session};
    const uint32_t box[4] = {(uint32_t)RK, 128, 1, 1};
    if ((s = make_map4(&maps[2], u->u, dims, str, box, vu_swizzle, "U")) != LRKV_OK) return s;
  }
  {  // B [N, r, Hkv*d]: box = 64 dims of one KV head x RK ranks of one agent, 128B-swizzled
     // (the B operand of the Z B MMA, d-major; ranks past p->rank arrive as zeros)
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p->num_kv_heads, (uint64_t)p->rank, (uint64_t)p->num_agents};
    const int64_t str[3] = {D, (int64_t)p->num_kv_heads * D, (int64_t)p->rank * p->num_kv_heads * D};
    const uint32_t box[4] = {64, 1, (uint32_t)RK, 1};
    if ((s = make_map4(&maps[3], b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, "B")) != LRKV_OK) return s;
  }
  lrkv::PrefillParams pp = {};
  pp.q = q;
  pp.offsets = alora_offsets;
  pp.page_table = kv->page_table;
  pp.pt_stride = kv->page_table_stride;
  pp.num_pages = kv->page_table ? kv->num_pages : 0;
  pp.out = out;
  pp.out_f32 = out_dtype == LRKV_F32;
  pp.N = p->num_agents;
  pp.Hq = p->num_q_heads;
  pp.Hkv = p->num_kv_heads;
  pp.G = G;
  pp.T = T;
  pp.L0 = ctx_len;
  pp.session = session;
  pp.mode = p->mode;
  pp.scale_log2 = scale_of(p) * 1.4426950408889634f;
  pp.flags = static_cast<unsigned*>(workspace);
  const lrkv::PrefillPlan pl = lrkv::plan_prefill(T, ctx_len, G, p->num_kv_heads, p->num_agents, D, dev.sms);
  if (workspace_bytes < pl.bytes)
    return fail(LRKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes (lrkv_prefill_workspace_bytes)", workspace_bytes, pl.bytes);
  pp.n_tb = pl.n_tb;
  pp.W_ga = pl.W_ga;
  pp.W = pl.W;
  pp.max_parts = pl.max_parts;
  pp.tickets = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + pl.tickets_off);
  pp.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.partials_off);
  take_stall_hook(&pp.spin_cap, &pp.stall);
  lrkv::PrefillMaps pm = {maps};
  s = lrkv::launch_prefill(pp, pm, D, RK, pl.ctas, stream);
  if (s != LRKV_OK) return fail(s, "prefill launch failed: %s", cudaGetErrorString(cudaGetLastError()));
  return LRKV_OK;
}

}  // extern "C"
