// pa_abi.cu -- the C ABI of libpa (declared in include/pa.h): argument validation,
// partition / group tables, TMA descriptors, workspace and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <utility>
#include <vector>

#include "../../include/pa.h"
#include "pa_device.cuh"
#include "pa_launch.h"

struct pa_ctx {
  int device = -1;
  int sm_count = 0;
  int* d_status = nullptr;         // device status word (bounded-wait give-ups)
  bool debug = false;              // PA_DEBUG: synchronise and check after every call
  void* ws = nullptr;              // workspace for per-block importance sums
  size_t ws_bytes = 0;
  std::string err;
};

namespace {

thread_local std::string g_init_err;

int fail(pa_ctx* ctx, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (ctx) ctx->err = buf; else g_init_err = buf;
  return code;
}

int cuda_fail(pa_ctx* ctx, int e, const char* what) {
  return fail(ctx, PA_ECUDA, "%s: %s", what, cudaGetErrorString(static_cast<cudaError_t>(e)));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Validate the partition table and build the group tables shared by the attention and
// merge paths.  fresh == NULL selects every pair.
int build_tables(pa_ctx* ctx, int N, int P, int G, const int32_t* part_off, const uint8_t* fresh,
                 pa::AttnTables& t) {
  if (P < 1 || P > PA_MAX_P) return fail(ctx, PA_EINVAL, "P=%d outside [1, %d]", P, PA_MAX_P);
  if (G < 1 || G > P) return fail(ctx, PA_EINVAL, "G=%d outside [1, P=%d]", G, P);
  if (!part_off) return fail(ctx, PA_EINVAL, "part_off is NULL");
  if (part_off[0] != 0) return fail(ctx, PA_EINVAL, "part_off[0]=%d, expected 0", part_off[0]);
  if (part_off[P] != N) return fail(ctx, PA_EINVAL, "part_off[P]=%d, expected N=%d", part_off[P], N);
  for (int p = 0; p < P; ++p)
    if (part_off[p + 1] < part_off[p])
      return fail(ctx, PA_EINVAL, "part_off decreases at %d (%d > %d)", p, part_off[p], part_off[p + 1]);
  memset(&t, 0, sizeof t);
  t.P = P;
  t.G = G;
  t.QG = (P + G - 1) / G;
  const int KG = t.QG;
  for (int p = 0; p <= P; ++p) t.part_off[p] = part_off[p];
  for (int g = 0; g <= t.QG; ++g) t.qg_row0[g] = part_off[g * G < P ? g * G : P];
  for (int qg = 0; qg < t.QG; ++qg)
    for (int p = 0; p < P; ++p) {
      const int kg = p / G;
      if (!fresh || fresh[qg * KG + kg]) t.fresh_bits[qg][p >> 5] |= 1u << (p & 31);
    }
  return PA_OK;
}

// Attention tiling: consecutive query groups that select the same fresh partitions form
// one segment, tiled as a unit (a row's states depend only on its own query and the
// partitions computed for it, so tiles may straddle such groups).  Replaces the group
// bounds and masks of `t` by the segments'.
void merge_equal_groups(pa::AttnTables& t) {
  int n = 0;
  for (int g = 0; g < t.QG; ++g) {
    if (n > 0 && memcmp(t.fresh_bits[n - 1], t.fresh_bits[g], sizeof t.fresh_bits[0]) == 0) continue;
    if (n != g) memcpy(t.fresh_bits[n], t.fresh_bits[g], sizeof t.fresh_bits[0]);
    t.qg_row0[n] = t.qg_row0[g];
    ++n;
  }
  t.qg_row0[n] = t.qg_row0[t.QG];
  for (int g = n; g < t.QG; ++g) memset(t.fresh_bits[g], 0, sizeof t.fresh_bits[0]);
  t.QG = n;
}

// Prefix of row tiles over the query groups that have at least one fresh pair.
int fill_tile_start(pa::AttnTables& t, int tile_rows) {
  int acc = 0;
  for (int qg = 0; qg < t.QG; ++qg) {
    t.tile_start[qg] = acc;
    bool any = false;
    for (int w = 0; w < PA_MAX_P / 32; ++w) any |= t.fresh_bits[qg][w] != 0;
    const int rows = t.qg_row0[qg + 1] - t.qg_row0[qg];
    if (any && rows > 0) acc += (rows + tile_rows - 1) / tile_rows;
  }
  t.tile_start[t.QG] = acc;
  return acc;
}

// Longest-first launch order for a bf16 attention grid of a few waves (more units than SMs,
// at most kMaxOrderedUnits): units sorted by their KV tile count, longest first, ties in
// unit order (stable).  Returns false, and leaves the grid in unit order, when every unit
// has the same length or the grid is one wave or very large: there the order cannot shorten
// the tail, and unit order keeps the CTAs of one head (which share K and V) together.
bool longest_first(const pa::TcParams& prm, int units, int sm_count, pa::TcUnitOrder& ord) {
  if (units <= sm_count || units > pa::kMaxOrderedUnits) return false;
  const pa::AttnTables& t = prm.t;
  int group_tiles[PA_MAX_P];
  for (int qg = 0; qg < t.QG; ++qg) {
    group_tiles[qg] = 0;
    for (int p = 0; p < t.P; ++p)
      if (pa::fresh_bit(t.fresh_bits, qg, p) && t.part_off[p + 1] > t.part_off[p])
        group_tiles[qg] += (t.part_off[p + 1] - t.part_off[p] + 127) / 128;
  }
  std::vector<std::pair<int, int>> key(units);        // (-tiles, unit)
  bool varied = false;
  for (int u = 0; u < units; ++u) {
    const int tix = u % prm.tiles_total;
    int qg = 0;
    while (qg + 1 < t.QG && t.tile_start[qg + 1] <= tix) ++qg;
    key[u] = {-group_tiles[qg], u};
    varied |= key[u].first != key[0].first;
  }
  if (!varied) return false;
  std::stable_sort(key.begin(), key.end());
  for (int i = 0; i < units; ++i) ord.unit[i] = static_cast<uint16_t>(key[i].second);
  return true;
}

// Host-side fault injection for tests (no GPU fault involved): PA_INJECT_ENOMEM, a
// comma-separated list of sites ("init", "workspace"), makes the named device allocations
// fail as if cudaMalloc had, without calling it.  Read at every allocation, so a process
// can arm and disarm it between calls.
bool inject_enomem(const char* site) {
  const char* env = getenv("PA_INJECT_ENOMEM");
  if (!env || !*env) return false;
  const size_t n = strlen(site);
  for (const char* p = env; *p;) {
    const char* end = strchr(p, ',');
    const size_t len = end ? static_cast<size_t>(end - p) : strlen(p);
    if (len == n && strncmp(p, site, n) == 0) return true;
    if (!end) break;
    p = end + 1;
  }
  return false;
}

int check_device(pa_ctx* ctx) {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaGetDevice");
  if (d != ctx->device)
    return fail(ctx, PA_EINVAL, "current device %d differs from the context's device %d", d, ctx->device);
  return PA_OK;
}

int ensure_ws(pa_ctx* ctx, size_t bytes) {
  if (bytes <= ctx->ws_bytes) return PA_OK;
  if (ctx->ws) {
    cudaFree(ctx->ws);
    ctx->ws = nullptr;
    ctx->ws_bytes = 0;
  }
  if (inject_enomem("workspace") || cudaMalloc(&ctx->ws, bytes) != cudaSuccess) {
    cudaGetLastError();
    ctx->ws = nullptr;
    return fail(ctx, PA_ENOMEM, "workspace allocation of %zu bytes failed", bytes);
  }
  ctx->ws_bytes = bytes;
  return PA_OK;
}

int encode_qkv_map(pa_ctx* ctx, CUtensorMap* m, const void* ptr, int BH, int N, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ctx, PA_ECUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ctx, PA_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PA_OK;
}

// Row blocks of the merge / importance kernels per (b, h) and their prefix per query group.
int fill_blk_start(const pa::AttnTables& t, int* blk_start) {
  const int rpb = pa::merge_rows_per_block();
  int acc = 0;
  for (int qg = 0; qg < t.QG; ++qg) {
    blk_start[qg] = acc;
    acc += (t.qg_row0[qg + 1] - t.qg_row0[qg] + rpb - 1) / rpb;
  }
  blk_start[t.QG] = acc;
  return acc;
}

int launch_reduce(pa_ctx* ctx, const pa::AttnTables& t, const int* blk_start, int blocks_per_bh, int BH,
                  const float* w_partial, float* w, cudaStream_t st) {
  pa::ReduceWParams r;
  memset(&r, 0, sizeof r);
  r.w_partial = w_partial;
  r.w = w;
  r.BH = BH;
  r.P = t.P;
  r.QG = t.QG;
  r.blocks_per_bh = blocks_per_bh;
  for (int g = 0; g <= t.QG; ++g) r.blk_start[g] = blk_start[g];
  for (int g = 0; g < t.QG; ++g) {
    const long long rows = t.qg_row0[g + 1] - t.qg_row0[g];
    r.inv_count[g] = rows > 0 ? 1.0 / (static_cast<double>(rows) * BH) : 0.0;
  }
  int e = pa::launch_reduce_w(r, st);
  return e ? cuda_fail(ctx, e, "reduce_w launch") : PA_OK;
}

// Argument checks and kernel parameters shared by pa_merge_states and
// pa_merge_states_noalloc: everything but the importance scratch (prm.w_partial stays
// null).  Errors are recorded on ctx (or, with ctx == NULL, in the thread's init-error
// slot that pa_last_error(NULL) reads).  *n_partials is the number of per-block importance
// sums the fused importance needs (0 without w); *launch is false when there is nothing to
// launch (N == 0).
int prepare_merge(pa_ctx* ctx, const pa_merge_desc* d, pa::AttnTables& t, pa::MergeParams& prm,
                  size_t* n_partials, bool* launch) {
  *launch = false;
  *n_partials = 0;
  if (!d) return fail(ctx, PA_EINVAL, "desc is NULL");
  if (d->dtype != PA_BF16 && d->dtype != PA_F32) return fail(ctx, PA_EUNSUPPORTED, "dtype %d", (int)d->dtype);
  if (d->D != 64 && d->D != 128) return fail(ctx, PA_EUNSUPPORTED, "D=%d (supported: 64, 128)", d->D);
  if (d->B < 1 || d->H < 1 || d->N < 0) return fail(ctx, PA_EINVAL, "B=%d H=%d N=%d", d->B, d->H, d->N);
  const long long BH = static_cast<long long>(d->B) * d->H;
  if (BH > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "B*H too large");
  int rc = build_tables(ctx, d->N, d->P, d->G, d->part_off, d->fresh, t);
  if (rc) return rc;
  bool all_fresh = true;
  for (int qg = 0; qg < t.QG; ++qg)
    for (int p = 0; p < t.P; ++p) all_fresh &= pa::fresh_bit(t.fresh_bits, qg, p);
  if (d->N == 0) return PA_OK;
  if (!d->o_fresh || !d->lse_fresh || !d->o || !d->lse) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!all_fresh && (!d->o_cached || !d->lse_cached))
    return fail(ctx, PA_EINVAL, "cached states are NULL but the mask reuses some pairs");
  if (d->cached_per_group != 0 && d->cached_per_group != 1)
    return fail(ctx, PA_EINVAL, "cached_per_group=%d (0 or 1)", d->cached_per_group);
  if (d->cached_per_group && d->w)
    return fail(ctx, PA_EINVAL, "importance needs per-partition cached states (w must be NULL with cached_per_group)");
  if (!aligned(d->o_fresh, 16) || !aligned(d->o, 16) || (d->o_cached && !aligned(d->o_cached, 16)))
    return fail(ctx, PA_EALIGN, "o_fresh, o_cached and o must be 16-byte aligned");
  if (!aligned(d->lse_fresh, 4) || !aligned(d->lse, 4) || (d->lse_cached && !aligned(d->lse_cached, 4)) ||
      (d->w && !aligned(d->w, 4)))
    return fail(ctx, PA_EALIGN, "lse arrays and w must be 4-byte aligned");
  memset(&prm, 0, sizeof prm);
  const int bpb = fill_blk_start(t, prm.blk_start);
  const long long blocks = BH * bpb;
  if (blocks > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "too many row blocks");
  prm.o_fresh = d->o_fresh;
  prm.lse_fresh = d->lse_fresh;
  prm.o_cached = d->o_cached;
  prm.lse_cached = d->lse_cached;
  prm.o = d->o;
  prm.lse = d->lse;
  prm.w_partial = nullptr;
  prm.BH = (int)BH;
  prm.N = d->N;
  prm.D = d->D;
  prm.P = t.P;
  prm.G = t.G;
  prm.QG = t.QG;
  prm.blocks_per_bh = bpb;
  prm.cached_per_group = d->cached_per_group;
  memcpy(prm.part_off, t.part_off, sizeof prm.part_off);
  memcpy(prm.qg_row0, t.qg_row0, sizeof prm.qg_row0);
  memcpy(prm.fresh_bits, t.fresh_bits, sizeof prm.fresh_bits);
  if (d->w) *n_partials = static_cast<size_t>(blocks) * t.P;
  *launch = true;
  return PA_OK;
}

}  // namespace

extern "C" {

const char* pa_version(void) { return "libpa 0.1 (sm_100a)"; }

int pa_init(int device, pa_ctx** out) {
  if (!out) return fail(nullptr, PA_EINVAL, "out is NULL");
  *out = nullptr;
  int n = 0;
  cudaError_t e = cudaGetDeviceCount(&n);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, PA_ECUDA, "cudaGetDeviceCount: %s", cudaGetErrorString(e));
  }
  if (device < 0 || device >= n) return fail(nullptr, PA_EINVAL, "device %d outside [0, %d)", device, n);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return fail(nullptr, PA_ECUDA, "cudaGetDeviceProperties: %s", cudaGetErrorString(e));
  if (prop.major != 10 || prop.minor != 0)
    return fail(nullptr, PA_EUNSUPPORTED, "device %d is sm_%d%d; libpa needs sm_100", device, prop.major,
                prop.minor);
  e = cudaSetDevice(device);
  if (e != cudaSuccess) return fail(nullptr, PA_ECUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
  pa_ctx* ctx = new pa_ctx();
  ctx->device = device;
  ctx->sm_count = prop.multiProcessorCount;
  const char* dbg = getenv("PA_DEBUG");
  ctx->debug = dbg && *dbg && strcmp(dbg, "0") != 0;
  if (inject_enomem("init") || cudaMalloc(&ctx->d_status, sizeof(int)) != cudaSuccess ||
      cudaMemset(ctx->d_status, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    if (ctx->d_status) cudaFree(ctx->d_status);
    delete ctx;
    return fail(nullptr, PA_ENOMEM, "status word allocation failed");
  }
  *out = ctx;
  return PA_OK;
}

void pa_destroy(pa_ctx* ctx) {
  if (!ctx) return;
  if (ctx->ws) cudaFree(ctx->ws);
  if (ctx->d_status) cudaFree(ctx->d_status);
  delete ctx;
}

const char* pa_last_error(const pa_ctx* ctx) { return ctx ? ctx->err.c_str() : g_init_err.c_str(); }

// Read and clear the context's status word once the stream's work is complete.
static int read_status(pa_ctx* ctx) {
  int h = 0;
  cudaError_t e = cudaMemcpy(&h, ctx->d_status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status read");
  if (h != 0) {
    cudaMemset(ctx->d_status, 0, sizeof(int));
    return fail(ctx, PA_ETIMEOUT, "a device-side wait gave up (status %d)", h);
  }
  return PA_OK;
}

int pa_sync_status(pa_ctx* ctx, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaStreamSynchronize");
  return read_status(ctx);
}

int pa_wait_status(pa_ctx* ctx, void* stream, double timeout_s) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (!(timeout_s >= 0.0) || timeout_s > 86400.0)
    return fail(ctx, PA_EINVAL, "timeout_s=%g outside [0, 86400]", timeout_s);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto t0 = std::chrono::steady_clock::now();
  const auto limit = std::chrono::duration<double>(timeout_s);
  auto nap = std::chrono::microseconds(20);
  while (true) {
    cudaError_t e = cudaStreamQuery(st);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return cuda_fail(ctx, e, "cudaStreamQuery");
    if (std::chrono::steady_clock::now() - t0 >= limit)
      return fail(ctx, PA_ETIMEOUT, "the stream's work did not finish within %g s (host deadline); "
                  "it was not cancelled and may be waited for again", timeout_s);
    std::this_thread::sleep_for(nap);
    if (nap < std::chrono::microseconds(2000)) nap *= 2;
  }
  return read_status(ctx);
}

static int pa_partition_attn_impl(pa_ctx* ctx, const pa_attn_desc* d, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (!d) return fail(ctx, PA_EINVAL, "desc is NULL");
  if (d->dtype != PA_BF16 && d->dtype != PA_F32) return fail(ctx, PA_EUNSUPPORTED, "dtype %d", (int)d->dtype);
  if (d->D != 64 && d->D != 128) return fail(ctx, PA_EUNSUPPORTED, "D=%d (supported: 64, 128)", d->D);
  if (d->B < 1 || d->H < 1 || d->N < 0) return fail(ctx, PA_EINVAL, "B=%d H=%d N=%d", d->B, d->H, d->N);
  const long long BH = static_cast<long long>(d->B) * d->H;
  if (BH > 65535) return fail(ctx, PA_EINVAL, "B*H=%lld exceeds 65535", BH);
  if (!(d->scale > 0.0f) || !(d->scale < 1e30f)) return fail(ctx, PA_EINVAL, "scale must be positive and finite");
  pa::AttnTables t;
  int rc = build_tables(ctx, d->N, d->P, d->G, d->part_off, d->fresh, t);
  if (rc) return rc;
  if (d->N == 0) return PA_OK;
  if (!d->q || !d->k || !d->v || !d->o_part || !d->lse_part)
    return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(d->q, 16) || !aligned(d->k, 16) || !aligned(d->v, 16) || !aligned(d->o_part, 16))
    return fail(ctx, PA_EALIGN, "q, k, v and o_part must be 16-byte aligned");
  if (!aligned(d->lse_part, 4)) return fail(ctx, PA_EALIGN, "lse_part must be 4-byte aligned");
  if ((rc = check_device(ctx))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (d->dtype == PA_BF16) {
    pa::TcParams prm;
    memset(&prm, 0, sizeof prm);
    prm.t = t;
    merge_equal_groups(prm.t);
    const int tiles = fill_tile_start(prm.t, pa::attn_tc_tile_rows());
    if (tiles == 0) return PA_OK;
    if ((rc = encode_qkv_map(ctx, &prm.tm_q, d->q, (int)BH, d->N, d->D))) return rc;
    if ((rc = encode_qkv_map(ctx, &prm.tm_k, d->k, (int)BH, d->N, d->D))) return rc;
    if ((rc = encode_qkv_map(ctx, &prm.tm_v, d->v, (int)BH, d->N, d->D))) return rc;
    prm.o_part = d->o_part;
    prm.lse_part = d->lse_part;
    prm.status = ctx->d_status;
    prm.BH = (int)BH;
    prm.N = d->N;
    prm.D = d->D;
    prm.tiles_total = tiles;
    prm.scale_log2 = d->scale * 1.4426950408889634f;
    const long long units = BH * tiles;
    if (units > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "too many work units");
    pa::TcUnitOrder order;
    const bool ordered = longest_first(prm, static_cast<int>(units), ctx->sm_count, order);
    int e = pa::launch_attn_tc(prm, ordered ? &order : nullptr, static_cast<int>(units), st);
    return e ? cuda_fail(ctx, e, "attn_tc launch") : PA_OK;
  }
  pa::F32AttnParams prm;
  memset(&prm, 0, sizeof prm);
  prm.t = t;
  merge_equal_groups(prm.t);
  const int tiles = fill_tile_start(prm.t, pa::attn_f32_tile_rows());
  if (tiles == 0) return PA_OK;
  prm.q = static_cast<const float*>(d->q);
  prm.k = static_cast<const float*>(d->k);
  prm.v = static_cast<const float*>(d->v);
  prm.o_part = static_cast<float*>(d->o_part);
  prm.lse_part = d->lse_part;
  prm.BH = (int)BH;
  prm.N = d->N;
  prm.D = d->D;
  prm.tiles_total = tiles;
  prm.scale = d->scale;
  int e = pa::launch_attn_f32(prm, st);
  return e ? cuda_fail(ctx, e, "attn_f32 launch") : PA_OK;
}

static int pa_merge_states_impl(pa_ctx* ctx, const pa_merge_desc* d, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  pa::AttnTables t;
  pa::MergeParams prm;
  size_t n_partials = 0;
  bool launch = false;
  int rc = prepare_merge(ctx, d, t, prm, &n_partials, &launch);
  if (rc || !launch) return rc;
  if ((rc = check_device(ctx))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->w) {
    if ((rc = ensure_ws(ctx, n_partials * sizeof(float)))) return rc;
    prm.w_partial = static_cast<float*>(ctx->ws);
  }
  int e = pa::launch_merge(prm, d->dtype, st);
  if (e) return cuda_fail(ctx, e, "merge launch");
  if (d->w) return launch_reduce(ctx, t, prm.blk_start, prm.blocks_per_bh, prm.BH, prm.w_partial, d->w, st);
  return PA_OK;
}

static int pa_compose_states_impl(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int factor,
                      const void* o_part, const float* lse_part, void* o_group, float* lse_group,
                      void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (dtype != PA_BF16 && dtype != PA_F32) return fail(ctx, PA_EUNSUPPORTED, "dtype %d", (int)dtype);
  if (D != 64 && D != 128) return fail(ctx, PA_EUNSUPPORTED, "D=%d (supported: 64, 128)", D);
  if (B < 1 || H < 1 || N < 0) return fail(ctx, PA_EINVAL, "B=%d H=%d N=%d", B, H, N);
  if (P < 1 || P > PA_MAX_P) return fail(ctx, PA_EINVAL, "P=%d outside [1, %d]", P, PA_MAX_P);
  if (factor < 1 || factor > P) return fail(ctx, PA_EINVAL, "factor=%d outside [1, P=%d]", factor, P);
  if (N == 0) return PA_OK;
  if (!o_part || !lse_part || !o_group || !lse_group) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(o_part, 16) || !aligned(o_group, 16)) return fail(ctx, PA_EALIGN, "o_part and o_group must be 16-byte aligned");
  if (!aligned(lse_part, 4) || !aligned(lse_group, 4)) return fail(ctx, PA_EALIGN, "lse arrays must be 4-byte aligned");
  int rc = check_device(ctx);
  if (rc) return rc;
  const long long BH = static_cast<long long>(B) * H;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pa::ComposeParams prm;
  memset(&prm, 0, sizeof prm);
  prm.o_part = o_part;
  prm.lse_part = lse_part;
  prm.o_group = o_group;
  prm.lse_group = lse_group;
  prm.BH = (int)BH;
  prm.N = N;
  prm.P = P;
  prm.factor = factor;
  const int rpb = pa::compose_rows_per_block();
  prm.nblk = (N + rpb - 1) / rpb;
  const long long C = (P + factor - 1) / factor;
  if (C * BH * prm.nblk > 0x7fffffffLL || BH > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "too many row blocks");
  int e = pa::launch_compose(prm, dtype, D, st);
  return e ? cuda_fail(ctx, e, "compose launch") : PA_OK;
}

static int pa_importance_impl(pa_ctx* ctx, int B, int H, int N, int P, int G, const int32_t* part_off,
                  const float* lse_part, const float* lse, float* w, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (B < 1 || H < 1 || N < 0) return fail(ctx, PA_EINVAL, "B=%d H=%d N=%d", B, H, N);
  pa::AttnTables t;
  int rc = build_tables(ctx, N, P, G, part_off, nullptr, t);
  if (rc) return rc;
  if (!w) return fail(ctx, PA_EINVAL, "w is NULL");
  if (N > 0 && (!lse_part || !lse)) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(lse_part, 4) || !aligned(lse, 4) || !aligned(w, 4))
    return fail(ctx, PA_EALIGN, "lse_part, lse and w must be 4-byte aligned");
  if ((rc = check_device(ctx))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long BH = static_cast<long long>(B) * H;
  pa::ImportanceParams prm;
  memset(&prm, 0, sizeof prm);
  const int bpb = fill_blk_start(t, prm.blk_start);
  const long long blocks = BH * bpb;
  if (blocks > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "too many row blocks");
  if (blocks > 0) {
    if ((rc = ensure_ws(ctx, static_cast<size_t>(blocks) * t.P * sizeof(float)))) return rc;
    prm.lse_part = lse_part;
    prm.lse = lse;
    prm.w_partial = static_cast<float*>(ctx->ws);
    prm.BH = (int)BH;
    prm.N = N;
    prm.P = t.P;
    prm.QG = t.QG;
    prm.blocks_per_bh = bpb;
    memcpy(prm.qg_row0, t.qg_row0, sizeof prm.qg_row0);
    int e = pa::launch_importance(prm, st);
    if (e) return cuda_fail(ctx, e, "importance launch");
  }
  return launch_reduce(ctx, t, prm.blk_start, bpb, (int)BH, static_cast<const float*>(ctx->ws), w, st);
}

static int pa_state_drift_impl(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int G,
                   const int32_t* part_off, const uint8_t* sel, const void* o_new, const void* o_ref,
                   float* d2, float* r2, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (dtype != PA_BF16 && dtype != PA_F32) return fail(ctx, PA_EINVAL, "unknown dtype %d", (int)dtype);
  if (B < 1 || H < 1 || N < 0) return fail(ctx, PA_EINVAL, "B=%d H=%d N=%d", B, H, N);
  if (D != 64 && D != 128) return fail(ctx, PA_EUNSUPPORTED, "D=%d (64 or 128 supported)", D);
  pa::AttnTables t;
  int rc = build_tables(ctx, N, P, G, part_off, nullptr, t);
  if (rc) return rc;
  if (!d2 || !r2) return fail(ctx, PA_EINVAL, "d2 or r2 is NULL");
  if (N > 0 && (!o_new || !o_ref)) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(o_new, 16) || !aligned(o_ref, 16) || !aligned(d2, 4) || !aligned(r2, 4))
    return fail(ctx, PA_EALIGN, "o_new and o_ref must be 16-byte aligned, d2 and r2 4-byte aligned");
  if ((rc = check_device(ctx))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "B*H too large");
  pa::DriftParams prm;
  memset(&prm, 0, sizeof prm);
  const int rpb = pa::drift_rows_per_block();
  int bpb = 0;
  for (int qg = 0; qg < t.QG; ++qg) {
    prm.blk_start[qg] = bpb;
    bpb += (t.qg_row0[qg + 1] - t.qg_row0[qg] + rpb - 1) / rpb;
  }
  prm.blk_start[t.QG] = bpb;
  const long long blocks = BH * bpb;
  if (blocks > 0x7fffffffLL) return fail(ctx, PA_EINVAL, "too many row blocks");
  if (blocks > 0) {
    if ((rc = ensure_ws(ctx, static_cast<size_t>(blocks) * 2 * t.P * sizeof(float)))) return rc;
    prm.o_new = o_new;
    prm.o_ref = o_ref;
    prm.partial = static_cast<float*>(ctx->ws);
    prm.BH = (int)BH;
    prm.N = N;
    prm.P = t.P;
    prm.G = t.G;
    prm.QG = t.QG;
    prm.blocks_per_bh = bpb;
    memcpy(prm.qg_row0, t.qg_row0, sizeof prm.qg_row0);
    for (int qg = 0; qg < t.QG; ++qg)
      for (int kg = 0; kg < t.QG; ++kg)
        if (!sel || sel[qg * t.QG + kg]) prm.sel_bits[qg][kg >> 5] |= 1u << (kg & 31);
    int e = pa::launch_drift(prm, dtype, D, st);
    if (e) return cuda_fail(ctx, e, "drift launch");
  }
  pa::ReducePairParams r;
  memset(&r, 0, sizeof r);
  r.partial = static_cast<const float*>(ctx->ws);
  r.d2 = d2;
  r.r2 = r2;
  r.BH = (int)BH;
  r.P = t.P;
  r.QG = t.QG;
  r.blocks_per_bh = bpb;
  memcpy(r.blk_start, prm.blk_start, sizeof r.blk_start);
  int e = pa::launch_reduce_pair(r, st);
  return e ? cuda_fail(ctx, e, "drift reduce launch") : PA_OK;
}

static int pa_selftest_wait_impl(pa_ctx* ctx, double seconds, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (!(seconds > 0.0 && seconds <= 2.0)) return fail(ctx, PA_EINVAL, "seconds=%g outside (0, 2]", seconds);
  int rc = check_device(ctx);
  if (rc) return rc;
  int e = pa::launch_wait_selftest(ctx->d_status, static_cast<uint64_t>(seconds * 1e9),
                                   static_cast<cudaStream_t>(stream));
  return e ? cuda_fail(ctx, e, "wait selftest launch") : PA_OK;
}

static int pa_relayout_seq2head_impl(pa_ctx* ctx, const void* src, void* dst, int N, int H, int D, int elem_bytes,
                         int n_chunks, int chunk, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (N < 0 || H < 1 || D < 1) return fail(ctx, PA_EINVAL, "N=%d H=%d D=%d", N, H, D);
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return fail(ctx, PA_EINVAL, "elem_bytes=%d", elem_bytes);
  const long long row_bytes = static_cast<long long>(D) * elem_bytes;
  if (row_bytes % 16 != 0) return fail(ctx, PA_EINVAL, "D*elem_bytes=%lld is not a multiple of 16", row_bytes);
  if (row_bytes > 16384) return fail(ctx, PA_EUNSUPPORTED, "D*elem_bytes=%lld above 16384", row_bytes);
  if (n_chunks < 1) return fail(ctx, PA_EINVAL, "n_chunks=%d", n_chunks);
  if (chunk < -1 || chunk >= n_chunks) return fail(ctx, PA_EINVAL, "chunk=%d outside [-1, %d)", chunk, n_chunks);
  if (N == 0) return PA_OK;
  if (!src || !dst) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(src, 16) || !aligned(dst, 16)) return fail(ctx, PA_EALIGN, "src and dst must be 16-byte aligned");
  int rc = check_device(ctx);
  if (rc) return rc;
  const long long step = (static_cast<long long>(N) + n_chunks - 1) / n_chunks;
  long long n0 = 0, n1 = N;
  if (chunk >= 0) {
    n0 = chunk * step < N ? chunk * step : N;
    n1 = (chunk + 1) * step < N ? (chunk + 1) * step : N;
  }
  int e = pa::launch_relayout(src, dst, n0, n1, n0, N, H, static_cast<int>(row_bytes), ctx->sm_count,
                              static_cast<cudaStream_t>(stream));
  return e ? cuda_fail(ctx, e, "relayout launch") : PA_OK;
}

static int pa_relayout_seq2head_at_impl(pa_ctx* ctx, const void* src, void* dst, int n_tok, int H, int D,
                                        int elem_bytes, int dst_tokens, int dst_tok0, void* stream) {
  if (!ctx) return fail(nullptr, PA_EINVAL, "ctx is NULL");
  if (n_tok < 0 || H < 1 || D < 1) return fail(ctx, PA_EINVAL, "n_tok=%d H=%d D=%d", n_tok, H, D);
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
    return fail(ctx, PA_EINVAL, "elem_bytes=%d", elem_bytes);
  const long long row_bytes = static_cast<long long>(D) * elem_bytes;
  if (row_bytes % 16 != 0) return fail(ctx, PA_EINVAL, "D*elem_bytes=%lld is not a multiple of 16", row_bytes);
  if (row_bytes > 16384) return fail(ctx, PA_EUNSUPPORTED, "D*elem_bytes=%lld above 16384", row_bytes);
  if (dst_tok0 < 0 || dst_tokens < 0 || static_cast<long long>(dst_tok0) + n_tok > dst_tokens)
    return fail(ctx, PA_EINVAL, "tokens [%d, %lld) outside the destination's %d", dst_tok0,
                static_cast<long long>(dst_tok0) + n_tok, dst_tokens);
  if (n_tok == 0) return PA_OK;
  if (!src || !dst) return fail(ctx, PA_EINVAL, "null tensor pointer");
  if (!aligned(src, 16) || !aligned(dst, 16)) return fail(ctx, PA_EALIGN, "src and dst must be 16-byte aligned");
  int rc = check_device(ctx);
  if (rc) return rc;
  int e = pa::launch_relayout(src, dst, 0, n_tok, dst_tok0, dst_tokens, H, static_cast<int>(row_bytes),
                              ctx->sm_count, static_cast<cudaStream_t>(stream));
  return e ? cuda_fail(ctx, e, "relayout launch") : PA_OK;
}

// With PA_DEBUG set when the context was created, every call synchronises its stream after
// launching and returns what pa_sync_status finds (a launch or runtime error, or a
// bounded device-side wait that gave up).
static int debug_finish(pa_ctx* ctx, void* stream, int rc) {
  if (rc != PA_OK || !ctx || !ctx->debug) return rc;
  return pa_sync_status(ctx, stream);
}

int pa_partition_attn(pa_ctx* ctx, const pa_attn_desc* d, void* stream) {
  return debug_finish(ctx, stream, pa_partition_attn_impl(ctx, d, stream));
}

int pa_merge_states(pa_ctx* ctx, const pa_merge_desc* d, void* stream) {
  return debug_finish(ctx, stream, pa_merge_states_impl(ctx, d, stream));
}

int pa_compose_states(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int factor,
                      const void* o_part, const float* lse_part, void* o_group, float* lse_group,
                      void* stream) {
  return debug_finish(ctx, stream, pa_compose_states_impl(ctx, dtype, B, H, N, D, P, factor, o_part, lse_part, o_group, lse_group, stream));
}

int pa_importance(pa_ctx* ctx, int B, int H, int N, int P, int G, const int32_t* part_off,
                  const float* lse_part, const float* lse, float* w, void* stream) {
  return debug_finish(ctx, stream, pa_importance_impl(ctx, B, H, N, P, G, part_off, lse_part, lse, w, stream));
}

int pa_state_drift(pa_ctx* ctx, pa_dtype dtype, int B, int H, int N, int D, int P, int G,
                   const int32_t* part_off, const uint8_t* sel, const void* o_new, const void* o_ref,
                   float* d2, float* r2, void* stream) {
  return debug_finish(ctx, stream, pa_state_drift_impl(ctx, dtype, B, H, N, D, P, G, part_off, sel, o_new, o_ref, d2, r2, stream));
}

int pa_relayout_seq2head(pa_ctx* ctx, const void* src, void* dst, int N, int H, int D, int elem_bytes,
                         int n_chunks, int chunk, void* stream) {
  return debug_finish(ctx, stream, pa_relayout_seq2head_impl(ctx, src, dst, N, H, D, elem_bytes, n_chunks, chunk, stream));
}

int pa_relayout_seq2head_at(pa_ctx* ctx, const void* src, void* dst, int n_tok, int H, int D, int elem_bytes,
                            int dst_tokens, int dst_tok0, void* stream) {
  return debug_finish(ctx, stream, pa_relayout_seq2head_at_impl(ctx, src, dst, n_tok, H, D, elem_bytes, dst_tokens,
                                                                dst_tok0, stream));
}

int pa_selftest_wait(pa_ctx* ctx, double seconds, void* stream) {
  return debug_finish(ctx, stream, pa_selftest_wait_impl(ctx, seconds, stream));
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free merge
// Scratch for pa_merge_states_noalloc: the per-block importance sums.  A file-scope device
// array, so every GPU that loads this library holds it (4 MiB) until the process exits.
// Host code must not use the symbol as a pointer: its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;   // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[128] = {};

int noalloc_scratch(int device, float** out) {
  if (device < 0 || device >= 128) return fail(nullptr, PA_EINVAL, "device %d outside [0, 128)", device);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return fail(nullptr, PA_ECUDA, "cudaGetSymbolAddress of the merge scratch failed on device %d: %s",
                  device, cudaGetErrorString(e));
    }
    g_noalloc_ptr[device] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[device];
  return PA_OK;
}

}  // namespace

extern "C" int pa_merge_states_noalloc(const pa_merge_desc* d, void* stream) {
  pa::AttnTables t;
  pa::MergeParams prm;
  size_t n_partials = 0;
  bool launch = false;
  int rc = prepare_merge(nullptr, d, t, prm, &n_partials, &launch);
  if (rc || !launch) return rc;
  float* scratch = nullptr;
  if (d->w) {
    if (n_partials > kNoAllocScratchFloats)
      return fail(nullptr, PA_EINVAL,
                  "importance scratch of %zu floats exceeds the fixed %zu (B*H*ceil(rows/128 per query "
                  "group)*P); use pa_merge_states",
                  n_partials, kNoAllocScratchFloats);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(nullptr, PA_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if ((rc = noalloc_scratch(dev, &scratch))) return rc;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prm.w_partial = scratch;
  int e = pa::launch_merge(prm, d->dtype, st);
  if (e) return fail(nullptr, PA_ECUDA, "merge launch: %s", cudaGetErrorString(static_cast<cudaError_t>(e)));
  if (!d->w) return PA_OK;
  return launch_reduce(nullptr, t, prm.blk_start, prm.blocks_per_bh, prm.BH, scratch, d->w, st);
}
