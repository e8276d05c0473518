// lod_api.cu -- the extern "C" entry points declared in include/lod.h:
// argument validation, index and workspace sizing, and kernel launches.
#include <atomic>
#include <initializer_list>
#include <utility>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "lod_internal.cuh"

namespace {

thread_local char g_err[512] = "";

int32_t fail(int32_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int32_t cuda_fail(cudaError_t e, const char* what) {
  return fail(LOD_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A per-call buffer the kernels read or write in place: memory of the current
// device, managed memory, or page-locked host memory mapped at the same
// address (cudaHostAlloc / cudaMallocHost under unified addressing: the
// kernels then move its bytes over the host link themselves).  Pageable host
// memory and another device's memory are refused before anything is enqueued.
int32_t check_visible(const void* ptr, const char* name, int* host = nullptr) {
  if (host) *host = 0;
  if (!ptr) return LOD_OK;
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, ptr);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(LOD_EINVAL, "%s: pointer not known to CUDA (%s)", name, cudaGetErrorString(e));
  }
  if (at.type == cudaMemoryTypeUnregistered)
    return fail(LOD_EINVAL, "%s is pageable host memory: pass device or page-locked host memory", name);
  if (at.type == cudaMemoryTypeHost && at.devicePointer != ptr)
    return fail(LOD_EINVAL, "%s: page-locked host memory not mapped at its host address", name);
  if (host) *host = at.type == cudaMemoryTypeHost;
  if (at.type == cudaMemoryTypeDevice) {
    int dev = -1;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (at.device != dev) return fail(LOD_EINVAL, "%s is memory of device %d, not the current device %d", name,
                                      at.device, dev);
  }
  return LOD_OK;
}

int32_t check_visible_all(std::initializer_list<std::pair<const void*, const char*>> bufs) {
  for (const auto& b : bufs) {
    const int32_t rc = check_visible(b.first, b.second);
    if (rc) return rc;
  }
  return LOD_OK;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t elem_bytes(const lod_params* p) { return p->dtype == LOD_DTYPE_F32 ? 4 : 2; }
int32_t page_slots(const lod_params* p) { return p->chunk / p->page + p->clusters; }
int32_t g_of(const lod_params* p) { return p->Hq / p->Hkv; }
// query rows per scan unit (registers: NQ x 8 fp32 accumulators per lane)
int nq_max(const lod_params*) { return 8; }

int32_t validate(const lod_params* p) {
  if (!p) return fail(LOD_EINVAL, "params is NULL");
  if (p->head_shard != 0) {
    const int tot = p->head_shard >> 16, first = p->head_shard & 0xffff;
    if (tot < p->Hkv || first + p->Hkv > tot)
      return fail(LOD_EINVAL, "head_shard: KV heads [%d, %d) outside the model's %d", first, first + p->Hkv, tot);
  }
  if (p->kv_bits != 0 && p->kv_bits != 4)
    return fail(LOD_EUNSUPPORTED, "kv_bits = %d unsupported (0 or 4)", p->kv_bits);
  if (p->kv_bits == 4 && p->top_pages == 0)
    return fail(LOD_EUNSUPPORTED, "three-tier INT4 (kv_bits = 4) needs top_pages >= 1");
  if (p->dtype != LOD_DTYPE_F32 && p->dtype != LOD_DTYPE_BF16)
    return fail(LOD_EUNSUPPORTED, "dtype %d unsupported (0=f32, 1=bf16)", p->dtype);
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1) return fail(LOD_EINVAL, "B, Hq, Hkv must be >= 1");
  if (p->Hq % p->Hkv) return fail(LOD_EINVAL, "Hq (%d) must be a multiple of Hkv (%d)", p->Hq, p->Hkv);
  const int g = g_of(p);
  if (g & (g - 1)) return fail(LOD_EUNSUPPORTED, "Hq/Hkv = %d must be a power of two", g);
  if (p->d != 64 && p->d != 128) return fail(LOD_EUNSUPPORTED, "d = %d unsupported (64 or 128)", p->d);
  if (g > nq_max(p)) return fail(LOD_EUNSUPPORTED, "Hq/Hkv = %d exceeds %d", g, nq_max(p));
  if (p->chunk != lod::kChunk) return fail(LOD_EUNSUPPORTED, "chunk must be %d", lod::kChunk);
  if (p->page != lod::kPage) return fail(LOD_EUNSUPPORTED, "page must be %d", lod::kPage);
  if (p->clusters < 1 || p->clusters > lod::kMaxClusters)
    return fail(LOD_EUNSUPPORTED, "clusters must be in [1, %d]", lod::kMaxClusters);
  if (p->kmeans_iters < 1 || p->kmeans_iters > 64)
    return fail(LOD_EUNSUPPORTED, "kmeans_iters must be in [1, 64]");
  if (p->top_groups < 1 || p->top_groups > lod::kMaxTopGroups)
    return fail(LOD_EUNSUPPORTED, "top_groups must be in [1, %d]", lod::kMaxTopGroups);
  if (p->top_pages < 0 || p->top_pages > lod::kMaxTopPages)
    return fail(LOD_EUNSUPPORTED, "top_pages must be in [0, %d] (0: two-tier LoD)", lod::kMaxTopPages);
  if (p->window < p->chunk || p->window % p->chunk)
    return fail(LOD_EINVAL, "window (%d) must be a positive multiple of chunk", p->window);
  if (p->sinks < 0 || p->sinks >= p->chunk) return fail(LOD_EINVAL, "sinks must be in [0, chunk)");
  if (p->Tmax < p->chunk || p->Tmax % p->chunk)
    return fail(LOD_EINVAL, "Tmax must be a positive multiple of chunk");
  if (p->Tmax / p->chunk * (int64_t)p->clusters > (int64_t)1 << 30)
    return fail(LOD_EUNSUPPORTED, "Tmax too large");
  return LOD_OK;
}

int32_t validate_kv(const lod_params* p, const void* K, const void* V, const int64_t* s) {
  if (!K || !V || !s) return fail(LOD_EINVAL, "K, V and kv_strides must be non-NULL");
  if (!aligned16(K) || !aligned16(V)) return fail(LOD_EINVAL, "K and V must be 16-byte aligned");
  const int64_t e = elem_bytes(p);
  for (int i = 0; i < 3; ++i)
    if (s[i] < 0 || (s[i] * e) % 16) return fail(LOD_EINVAL, "kv stride %d must be a non-negative multiple of 16 bytes", i);
  if (s[2] < p->d) return fail(LOD_EINVAL, "token stride smaller than d");
  return LOD_OK;
}

int32_t validate_index(const lod_params* p, const lod_index* ix) {
  if (!ix) return fail(LOD_EINVAL, "index is NULL");
  const void* ptrs[LOD_INDEX_ARRAYS] = {ix->gK,   ix->gV,    ix->gCnt, ix->pK, ix->pV,    ix->pCnt,
                                        ix->pBeg, ix->gPage, ix->perm, ix->mK, ix->mV,    ix->gMeta,
                                        ix->qK,   ix->qV,    ix->qKs,  ix->qVs};
  const bool int4 = p->kv_bits == 4;
  for (int i = 0; i < LOD_INDEX_ARRAYS; ++i) {
    const bool used = (i == 9 || i == 10) ? !int4 : (i >= 12 ? int4 : true);
    if (!used) continue;
    if (!ptrs[i]) return fail(LOD_EINVAL, "index field %d is NULL", i);
    if (i == 0 || i == 1 || i == 3 || i == 4 || i == 9 || i == 10 || i >= 12) {
      if (!aligned16(ptrs[i])) return fail(LOD_EINVAL, "index summary %d must be 16-byte aligned", i);
    } else if (i == 8) {
      if (!aligned16(ptrs[i])) return fail(LOD_EINVAL, "index member list (perm) must be 16-byte aligned");
    } else if ((i == 2 || i == 5 || i == 11) && (reinterpret_cast<uintptr_t>(ptrs[i]) & 3u)) {
      return fail(LOD_EINVAL, "index field %d misaligned", i);
    } else if (reinterpret_cast<uintptr_t>(ptrs[i]) & 1u) {
      return fail(LOD_EINVAL, "index field %d misaligned", i);
    }
  }
  return LOD_OK;
}

struct AttendShape {
  int NQ, NP, nsplit;
  int64_t units;
  bool tc;  // tensor-core scan (bf16, d = 128)
};

// Splits per unit: enough scan CTAs to fill the GPU (`target` CTAs), never
// fewer than one pipeline stage of rows per split.
int split_count(int64_t units, int64_t rows, int64_t target, int64_t rows_per_stage) {
  int64_t s = units >= target ? 1 : target / units;
  const int64_t most = cdiv(rows, rows_per_stage);
  if (s > most) s = most;
  if (s < 1) s = 1;
  return (int)s;
}

// Longest row list of a unit: every group of the index and the window.
int64_t max_rows(const lod_params* p) { return p->Tmax / p->chunk * p->clusters + p->window; }

// The tensor-core scan runs for bf16 caches with d = 128 (one CTA per SM,
// 128-row tiles, up to 16 query rows per unit); everything else takes the
// CUDA-core scan (two CTAs per SM, 64-row stages, up to 8 query rows).
bool use_tc(const lod_params* p) {
  return p->dtype == LOD_DTYPE_BF16 && p->d == 128 &&
         (int64_t)p->B * p->Hkv * (p->Tmax / p->chunk) * p->clusters < ((int64_t)1 << 31) &&
         p->Tmax < ((int64_t)1 << 31);
}
constexpr int64_t kTcCtas = 148, kTcTile = 128, kCoreCtas = lod::kTargetCtas;

int split_for(const lod_params* p, bool tc, int64_t units, int64_t rows) {
  return tc ? split_count(units, rows, kTcCtas, kTcTile) : split_count(units, rows, kCoreCtas, lod::kScanSlab);
}

// Decode: one unit per (b, kvh).
AttendShape decode_shape(const lod_params* p) {
  AttendShape s;
  s.tc = use_tc(p);
  s.NP = 1;
  s.NQ = g_of(p);
  s.units = (int64_t)p->B * p->Hkv;
  s.nsplit = split_for(p, s.tc, s.units, max_rows(p));
  return s;
}

// Prefill: one launch per query chunk; NP positions per unit.
AttendShape prefill_shape(const lod_params* p) {
  AttendShape s;
  s.tc = use_tc(p);
  s.NP = nq_max(p) / g_of(p);
  s.NQ = s.NP * g_of(p);
  s.units = (int64_t)p->B * p->Hkv * cdiv(p->chunk, s.NP);
  s.nsplit = split_for(p, s.tc, s.units, max_rows(p));
  return s;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int32_t encode_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, cuuint32_t box_rows = 128) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(LOD_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint32_t box4[4] = {64, box_rows, 1, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
                        strides_bytes, box4, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LOD_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LOD_OK;
}

// Tensor maps of the group summaries and the KV cache for the tensor-core scan.
int32_t make_tc_maps(const lod_params* p, const void* K, const void* V, const int64_t* kv, const lod_index* ix,
                     lod::TcMaps* m) {
  const cuuint64_t rows = (cuuint64_t)p->B * p->Hkv * (p->Tmax / p->chunk) * p->clusters;
  const cuuint64_t gdims[2] = {(cuuint64_t)p->d, rows};
  const cuuint64_t gstr[1] = {(cuuint64_t)p->d * 2};
  int32_t rc = encode_map(&m->gK, ix->gK, 2, gdims, gstr);
  if (!rc) rc = encode_map(&m->gV, ix->gV, 2, gdims, gstr);
  const cuuint64_t kdims[4] = {(cuuint64_t)p->d, (cuuint64_t)p->Tmax, (cuuint64_t)p->Hkv, (cuuint64_t)p->B};
  const cuuint64_t kstr[3] = {(cuuint64_t)kv[2] * 2, (cuuint64_t)kv[1] * 2, (cuuint64_t)kv[0] * 2};
  if (!rc) rc = encode_map(&m->K, K, 4, kdims, kstr);
  if (!rc) rc = encode_map(&m->V, V, 4, kdims, kstr);
  return rc;
}

// ---------------------------------------------------------------- grouped prefill

// The grouped tensor-core prefill runs for bf16 caches with d = 128 and the
// cache-dtype member copies (kv_bits = 0), when every row index it forms
// fits in 32 bits.
bool use_tc_prefill(const lod_params* p) {
  const int64_t Cmax = p->Tmax / p->chunk;
  return use_tc(p) && p->kv_bits == 0 && (int64_t)p->B * p->Hkv * p->Tmax < ((int64_t)1 << 31) &&
         (int64_t)p->B * p->Hq * p->Tmax < ((int64_t)1 << 31) &&
         (int64_t)p->B * p->Hkv * Cmax * page_slots(p) < ((int64_t)1 << 31);
}

constexpr int kItemRows = 1024;                    // pairs per work item of the pair kernel
constexpr int64_t kPrefillWaveBudget = (int64_t)2 << 30;  // workspace bytes a wave may use

// Workspace bytes per wave row: state (132 floats), and per opened group
// its id, its coarse weight, its place in the group's run, its log-sum-exp,
// its bf16 output and its two pair-list entries (pair id, row of q).
int64_t pf_row_bytes(const lod_params* p) { return 132 * 4 + (int64_t)p->top_groups * (4 + 4 + 4 + 4 + 2 * p->d + 4 + 4); }

// Query positions per wave: a multiple of chunk, as many as the budget allows
// (at least one chunk, at most 128), never more than the cache holds.
int64_t pf_wave(const lod_params* p) {
  const int64_t rows = (int64_t)p->B * p->Hq;
  int64_t nw = kPrefillWaveBudget / (rows * pf_row_bytes(p)) / p->chunk * p->chunk;
  const int64_t most = (((int64_t)1 << 31) - 1) / (rows * p->top_groups) / p->chunk * p->chunk;
  if (nw > most) nw = most;
  if (nw > 128 * (int64_t)p->chunk) nw = 128 * (int64_t)p->chunk;
  if (nw > p->Tmax) nw = p->Tmax;
  if (nw < p->chunk) nw = p->chunk;
  return nw;
}

struct PfLayout {
  size_t state, sel, cw, pos, plse, po, list, list_q, cnt, off, items, n_items, total;
  int64_t NW, Gtot, max_items;
};

PfLayout pf_layout(const lod_params* p) {
  PfLayout L;
  L.NW = pf_wave(p);
  const int64_t rows = (int64_t)p->B * p->Hq * L.NW;
  const int64_t pairs = rows * p->top_groups;
  L.Gtot = (int64_t)p->B * p->Hkv * (p->Tmax / p->chunk) * p->clusters;
  L.max_items = pairs / kItemRows + L.Gtot + 1;
  size_t o = lod::kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += (bytes + 255) & ~size_t(255);
    return at;
  };
  L.state = take(sizeof(float) * 132 * (size_t)rows);
  L.sel = take(sizeof(int32_t) * (size_t)pairs);
  L.cw = take(sizeof(float) * (size_t)pairs);
  L.pos = take(sizeof(int32_t) * (size_t)pairs);
  L.plse = take(sizeof(float) * (size_t)pairs);
  L.po = take((size_t)2 * p->d * (size_t)pairs);
  L.list = take(sizeof(int32_t) * (size_t)pairs);
  L.list_q = take(sizeof(int32_t) * (size_t)pairs);
  L.cnt = take(sizeof(int32_t) * (size_t)L.Gtot);
  L.off = take(sizeof(int32_t) * (size_t)L.Gtot);
  L.items = take(16 * 2 * (size_t)L.max_items);  // small-group items, then large-group items
  L.n_items = take(16);
  L.total = o;
  return L;
}

int g_num_sms[64] = {};

// A second stream of the current device for work that overlaps the caller's
// stream inside one call (created once per device, never destroyed; it only
// ever waits on events of the caller's stream).
cudaStream_t g_side[64] = {};
std::mutex g_side_mu;

int32_t side_stream(cudaStream_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LOD_EUNSUPPORTED, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lk(g_side_mu);
  if (!g_side[dev]) {
    e = cudaStreamCreateWithFlags(&g_side[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
  }
  *out = g_side[dev];
  return LOD_OK;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!g_num_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

// Tensor maps of the pair kernel: member-ordered copies and page summaries.
int32_t make_pair_maps(const lod_params* p, const lod_index* ix, lod::PairMaps* m) {
  const cuuint64_t Cmax = (cuuint64_t)(p->Tmax / p->chunk);
  const cuuint64_t mrows = (cuuint64_t)p->B * p->Hkv * Cmax * p->chunk;
  const cuuint64_t prows = (cuuint64_t)p->B * p->Hkv * Cmax * page_slots(p);
  const cuuint64_t str[1] = {(cuuint64_t)p->d * 2};
  const cuuint64_t md[2] = {(cuuint64_t)p->d, mrows}, pd[2] = {(cuuint64_t)p->d, prows};
  int32_t rc = encode_map(&m->mK, ix->mK, 2, md, str, 32);
  if (!rc) rc = encode_map(&m->mV, ix->mV, 2, md, str, 32);
  if (!rc) rc = encode_map(&m->pK, ix->pK, 2, pd, str, 16);
  if (!rc) rc = encode_map(&m->pV, ix->pV, 2, pd, str, 16);
  return rc;
}

// Workspace of a scan/refine pair: the split states, then either every
// group's score per query row (CUDA-core scan) or each split's best groups
// per query row (tensor-core scan).
size_t attend_ws_bytes(const lod_params* p, const AttendShape& s) {
  size_t part = sizeof(float) * (size_t)s.units * s.nsplit * s.NQ * (p->d + 2);
  size_t sel = s.tc ? sizeof(lod::SplitCand) * (size_t)s.units * s.nsplit * s.NQ * p->top_groups
                    : sizeof(float2) * (size_t)s.units * s.NQ * (size_t)(p->Tmax / p->chunk) * p->clusters;
  return lod::kWsHeader + ((part + 255) & ~size_t(255)) + ((sel + 255) & ~size_t(255));
}

void fill_attend(lod::AttendArgs& a, const lod_params* p, const AttendShape& s, const void* K,
                 const void* V, const int64_t* kv, const lod_index* ix, void* ws) {
  memset(&a, 0, sizeof(a));
  a.K = K;
  a.V = V;
  a.sb = kv[0];
  a.sh = kv[1];
  a.st = kv[2];
  a.gK = ix->gK;
  a.gV = ix->gV;
  a.gCnt = ix->gCnt;
  a.pK = ix->pK;
  a.pV = ix->pV;
  a.pCnt = ix->pCnt;
  a.pBeg = ix->pBeg;
  a.gPage = ix->gPage;
  a.perm = ix->perm;
  a.mK = ix->mK;
  a.mV = ix->mV;
  a.gMeta = ix->gMeta;
  a.kv_bits = p->kv_bits;
  a.qK = ix->qK;
  a.qV = ix->qV;
  a.qKs = reinterpret_cast<const float2*>(ix->qKs);
  a.qVs = reinterpret_cast<const float2*>(ix->qVs);
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.g = g_of(p);
  a.Tmax = p->Tmax;
  a.Cmax = p->Tmax / p->chunk;
  a.k = p->clusters;
  a.P = page_slots(p);
  a.G = p->top_groups;
  a.TP = p->top_pages;
  a.window = p->window;
  a.sinks = p->sinks;
  a.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
  a.NP = s.NP;
  a.nsplit = s.nsplit;
  a.units = s.units;
  char* w = static_cast<char*>(ws);
  a.status = reinterpret_cast<uint32_t*>(w);
  size_t part = sizeof(float) * (size_t)s.units * s.nsplit * s.NQ * (p->d + 2);
  part = (part + 255) & ~size_t(255);
  a.part = reinterpret_cast<float*>(w + lod::kWsHeader);
  if (s.tc)
    a.cand = reinterpret_cast<lod::SplitCand*>(w + lod::kWsHeader + part);
  else
    a.gsc = reinterpret_cast<float2*>(w + lod::kWsHeader + part);
}

int32_t do_build(const lod_params* p, const void* K, const void* V, const int64_t* kv, int64_t c0,
                 int64_t c1, const lod_index* ix, void* ws, cudaStream_t stream,
                 const int64_t* seq_lens = nullptr) {
  lod::BuildArgs a;
  memset(&a, 0, sizeof(a));
  a.K = K;
  a.V = V;
  a.sb = kv[0];
  a.sh = kv[1];
  a.st = kv[2];
  a.Hkv = p->Hkv;
  a.Cmax = p->Tmax / p->chunk;
  a.k = p->clusters;
  a.iters = p->kmeans_iters;
  a.sinks = p->sinks;
  a.head_shard = p->head_shard;
  a.P = page_slots(p);
  a.chunk_begin = c0;
  a.seq_lens = seq_lens;
  a.seed = p->seed;
  a.gK = ix->gK;
  a.gV = ix->gV;
  a.gCnt = ix->gCnt;
  a.pK = ix->pK;
  a.pV = ix->pV;
  a.pCnt = ix->pCnt;
  a.pBeg = ix->pBeg;
  a.gPage = ix->gPage;
  a.perm = ix->perm;
  a.mK = ix->mK;
  a.mV = ix->mV;
  a.gMeta = ix->gMeta;
  a.kv_bits = p->kv_bits;
  a.qK = ix->qK;
  a.qV = ix->qV;
  a.qKs = reinterpret_cast<float2*>(ix->qKs);
  a.qVs = reinterpret_cast<float2*>(ix->qVs);
  a.status = static_cast<uint32_t*>(ws);
  cudaError_t e = lod::launch_build(a, p->dtype, p->d, c1 - c0, p->B, stream);
  if (e != cudaSuccess) return cuda_fail(e, "index build launch");
  return LOD_OK;
}

}  // namespace

extern "C" {

int32_t lod_version(void) { return 100; }

const char* lod_last_error(void) { return g_err; }

int32_t lod_index_sizes(const lod_params* p, size_t bytes[LOD_INDEX_ARRAYS]) {
  int32_t rc = validate(p);
  if (rc) return rc;
  if (!bytes) return fail(LOD_EINVAL, "bytes is NULL");
  const size_t units = (size_t)p->B * p->Hkv, Cmax = p->Tmax / p->chunk, k = p->clusters,
               P = page_slots(p), d = p->d, e = elem_bytes(p);
  bytes[0] = bytes[1] = units * Cmax * k * d * e;
  bytes[2] = units * Cmax * k * sizeof(int32_t);
  bytes[3] = bytes[4] = units * Cmax * P * d * e;
  bytes[5] = units * Cmax * P * sizeof(int32_t);
  bytes[6] = units * Cmax * P * sizeof(int16_t);
  bytes[7] = units * Cmax * (k + 1) * sizeof(int16_t);
  bytes[8] = units * Cmax * p->chunk * sizeof(int16_t);
  const bool int4 = p->kv_bits == 4;
  bytes[9] = bytes[10] = int4 ? 0 : units * Cmax * p->chunk * d * e;
  bytes[11] = units * Cmax * k * sizeof(int32_t);
  bytes[12] = bytes[13] = int4 ? units * Cmax * p->chunk * d / 2 : 0;
  bytes[14] = bytes[15] = int4 ? units * Cmax * P * d * 2 * sizeof(float) : 0;
  g_err[0] = 0;
  return LOD_OK;
}

int32_t lod_workspace_bytes(const lod_params* p, int32_t op, size_t* bytes) {
  int32_t rc = validate(p);
  if (rc) return rc;
  if (!bytes) return fail(LOD_EINVAL, "bytes is NULL");
  switch (op) {
    case LOD_OP_BUILD: *bytes = lod::kWsHeader; break;
    case LOD_OP_DECODE: *bytes = attend_ws_bytes(p, decode_shape(p)); break;
    case LOD_OP_PREFILL: {
      // the grouped path's waves, or the per-chunk path (q in host memory)
      size_t b = attend_ws_bytes(p, prefill_shape(p));
      if (use_tc_prefill(p)) {
        const size_t t = pf_layout(p).total;
        if (t > b) b = t;
      }
      *bytes = b;
      break;
    }
    default: return fail(LOD_EINVAL, "unknown op %d", op);
  }
  g_err[0] = 0;
  return LOD_OK;
}

int32_t lod_build_index(const lod_params* p, const void* K, const void* V, const int64_t kv_strides[3],
                        int64_t chunk_begin, int64_t chunk_end, const lod_index* index, void* ws,
                        size_t ws_bytes, lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (!rc) rc = validate_index(p, index);
  if (rc) return rc;
  if (chunk_begin < 0 || chunk_end <= chunk_begin || chunk_end * p->chunk > p->Tmax)
    return fail(LOD_EINVAL, "chunk range [%lld, %lld) invalid for Tmax %lld", (long long)chunk_begin,
                (long long)chunk_end, (long long)p->Tmax);
  if (chunk_end - chunk_begin > 0x7fffffff) return fail(LOD_EINVAL, "chunk range too large");
  if (!ws || !aligned16(ws) || ws_bytes < lod::kWsHeader)
    return fail(LOD_EINVAL, "workspace too small or misaligned");
  rc = do_build(p, K, V, kv_strides, chunk_begin, chunk_end, index, ws, (cudaStream_t)stream);
  if (!rc) g_err[0] = 0;
  return rc;
}

int32_t lod_append_kv(const lod_params* p, void* K, void* V, const int64_t kv_strides[3], const int64_t* seq_lens,
                      const void* k_new, const void* v_new, lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (rc) return rc;
  if (!seq_lens || !k_new || !v_new) return fail(LOD_EINVAL, "seq_lens, k_new and v_new must be non-NULL");
  if (!aligned16(k_new) || !aligned16(v_new)) return fail(LOD_EINVAL, "k_new and v_new must be 16-byte aligned");
  rc = check_visible_all({{seq_lens, "seq_lens"}, {k_new, "k_new"}, {v_new, "v_new"}});
  if (rc) return rc;
  cudaError_t e = lod::launch_append(K, V, kv_strides, (int)elem_bytes(p), p->d, seq_lens, k_new, v_new, p->B,
                                     p->Hkv, p->Tmax, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  g_err[0] = 0;
  return LOD_OK;
}

int32_t lod_build_ready(const lod_params* p, const void* K, const void* V, const int64_t kv_strides[3],
                        const int64_t* seq_lens, const lod_index* index, void* ws, size_t ws_bytes,
                        lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (!rc) rc = validate_index(p, index);
  if (rc) return rc;
  if (!seq_lens) return fail(LOD_EINVAL, "seq_lens must be non-NULL");
  if (!ws || !aligned16(ws) || ws_bytes < lod::kWsHeader)
    return fail(LOD_EINVAL, "workspace too small or misaligned");
  rc = do_build(p, K, V, kv_strides, 0, 1, index, ws, (cudaStream_t)stream, seq_lens);
  if (!rc) g_err[0] = 0;
  return rc;
}

int32_t lod_decode(const lod_params* p, const void* q, const void* K, const void* V,
                   const int64_t kv_strides[3], const int64_t* seq_lens, const lod_index* index,
                   void* out, float* lse, int32_t* sel_groups, int32_t* sel_pages, void* ws,
                   size_t ws_bytes, lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (!rc) rc = validate_index(p, index);
  if (rc) return rc;
  if (!q || !out || !seq_lens) return fail(LOD_EINVAL, "q, out and seq_lens must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(LOD_EINVAL, "q and out must be 16-byte aligned");
  const AttendShape s = decode_shape(p);
  if (!ws || !aligned16(ws) || ws_bytes < attend_ws_bytes(p, s))
    return fail(LOD_EINVAL, "workspace too small (%zu < %zu) or misaligned", ws_bytes, attend_ws_bytes(p, s));
  int q_host = 0;
  rc = check_visible(q, "q", &q_host);
  if (!rc) rc = check_visible_all({{out, "out"}, {seq_lens, "seq_lens"}, {lse, "lse"},
                                   {sel_groups, "sel_groups"}, {sel_pages, "sel_pages"}});
  if (rc) return rc;
  lod::AttendArgs a;
  fill_attend(a, p, s, K, V, kv_strides, index, ws);
  a.q = q;
  a.q_host = q_host;
  a.Tq = 1;
  a.q_begin = 0;
  a.seq_lens = seq_lens;
  a.pos_lo = 0;
  a.pos_hi = 1;
  a.out = out;
  a.lse = lse;
  a.sel_groups = sel_groups;
  a.sel_pages = sel_pages;
  lod::TcMaps maps;
  if (s.tc) {
    rc = make_tc_maps(p, K, V, kv_strides, index, &maps);
    if (rc) return rc;
  }
  cudaError_t e = lod::launch_attend(a, p->dtype, p->d, s.NQ, s.tc ? &maps : nullptr, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  g_err[0] = 0;
  return LOD_OK;
}

int32_t lod_prefill(const lod_params* p, const void* q, int64_t q_begin, int64_t Tq, const void* K,
                    const void* V, const int64_t kv_strides[3], const lod_index* index, void* out,
                    float* lse, int32_t* sel_groups, int32_t* sel_pages, void* ws, size_t ws_bytes,
                    lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (!rc) rc = validate_index(p, index);
  if (rc) return rc;
  if (!q || !out) return fail(LOD_EINVAL, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(LOD_EINVAL, "q and out must be 16-byte aligned");
  if (q_begin < 0 || q_begin % p->chunk || Tq < 1 || q_begin + Tq > p->Tmax)
    return fail(LOD_EINVAL, "query range [%lld, %lld) invalid", (long long)q_begin, (long long)(q_begin + Tq));
  const AttendShape s = prefill_shape(p);
  if (!ws || !aligned16(ws) || ws_bytes < attend_ws_bytes(p, s))
    return fail(LOD_EINVAL, "workspace too small (%zu < %zu) or misaligned", ws_bytes, attend_ws_bytes(p, s));
  int q_host = 0;
  rc = check_visible(q, "q", &q_host);
  if (!rc) rc = check_visible_all({{out, "out"}, {lse, "lse"}, {sel_groups, "sel_groups"},
                                   {sel_pages, "sel_pages"}});
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t c0 = q_begin / p->chunk, c1 = (q_begin + Tq) / p->chunk;
  if (use_tc_prefill(p) && !q_host) {
    // 2) grouped tensor-core attention, one wave of query chunks at a time
    const PfLayout L = pf_layout(p);
    lod::TcMaps maps;
    lod::PairMaps pmaps;
    rc = make_tc_maps(p, K, V, kv_strides, index, &maps);
    if (!rc) rc = make_pair_maps(p, index, &pmaps);
    if (rc) return rc;
    char* w = static_cast<char*>(ws);
    lod::PrefillArgs a;
    memset(&a, 0, sizeof(a));
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.Tq = Tq;
    a.q_begin = q_begin;
    a.B = p->B;
    a.Hq = p->Hq;
    a.Hkv = p->Hkv;
    a.g = g_of(p);
    a.Tmax = p->Tmax;
    a.Cmax = p->Tmax / p->chunk;
    a.k = p->clusters;
    a.P = page_slots(p);
    a.G = p->top_groups;
    a.TP = p->top_pages;
    a.window = p->window;
    a.sinks = p->sinks;
    a.scale_log2 = (p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d)) * 1.4426950408889634f;
    a.gMeta = index->gMeta;
    a.gV = static_cast<const __nv_bfloat16*>(index->gV);
    a.pBeg = index->pBeg;
    a.pCnt = index->pCnt;
    a.NW = L.NW;
    a.state = reinterpret_cast<float*>(w + L.state);
    a.sel = reinterpret_cast<int32_t*>(w + L.sel);
    a.cw = reinterpret_cast<float*>(w + L.cw);
    a.pos = reinterpret_cast<int32_t*>(w + L.pos);
    a.plse = reinterpret_cast<float*>(w + L.plse);
    a.po = reinterpret_cast<__nv_bfloat16*>(w + L.po);
    a.list = reinterpret_cast<int32_t*>(w + L.list);
    a.list_q = reinterpret_cast<int32_t*>(w + L.list_q);
    a.cnt = reinterpret_cast<int32_t*>(w + L.cnt);
    a.off = reinterpret_cast<int32_t*>(w + L.off);
    a.items = reinterpret_cast<int4*>(w + L.items);
    a.big_items = L.max_items;
    a.n_items = reinterpret_cast<int32_t*>(w + L.n_items);
    a.Gtot = L.Gtot;
    a.item_rows = kItemRows;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.sel_groups = sel_groups;
    a.sel_pages = sel_pages;
    a.status = reinterpret_cast<uint32_t*>(w);
    const int nsm = num_sms();
    // The index of the chunks a wave completes is built before the wave
    // attends; the next wave's chunks are built on a second stream while
    // this wave attends.  Its queries see a chunk only window/chunk chunks
    // after it completes, so no wave reads a chunk that is being built.
    auto wave_chunks = [&](int64_t lo, int64_t hi, int64_t& b0, int64_t& b1) {
      b0 = (q_begin + lo) / p->chunk;
      b1 = (q_begin + hi) / p->chunk;
    };
    cudaStream_t side = nullptr;
    cudaEvent_t ev[2] = {nullptr, nullptr};
    if (Tq > L.NW) {
      rc = side_stream(&side);
      if (!rc && cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming) != cudaSuccess) rc = fail(LOD_ECUDA, "event");
      if (!rc && cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) != cudaSuccess) rc = fail(LOD_ECUDA, "event");
      if (rc) {
        if (ev[0]) cudaEventDestroy(ev[0]);
        return rc;
      }
    }
    auto done = [&](int32_t code) {
      for (cudaEvent_t e : ev)
        if (e) cudaEventDestroy(e);  // (released once their work has completed)
      return code;
    };
    int64_t b0, b1;
    wave_chunks(0, L.NW < Tq ? L.NW : Tq, b0, b1);
    if (b1 > b0) {
      rc = do_build(p, K, V, kv_strides, b0, b1, index, ws, st);
      if (rc) return done(rc);
    }
    int k = 0;
    for (int64_t lo = 0; lo < Tq; lo += L.NW, k ^= 1) {
      a.w_lo = lo;
      a.w_hi = lo + L.NW < Tq ? lo + L.NW : Tq;
      const int64_t nlo = a.w_hi, nhi = nlo + L.NW < Tq ? nlo + L.NW : Tq;
      bool built_next = false;
      if (nlo < Tq) {  // the next wave's chunks, on the second stream
        wave_chunks(nlo, nhi, b0, b1);
        if (b1 > b0) {
          cudaError_t e = cudaEventRecord(ev[k], st);
          if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev[k], 0);
          if (e != cudaSuccess) return done(cuda_fail(e, "prefill stream fork"));
          rc = do_build(p, K, V, kv_strides, b0, b1, index, ws, side);
          if (rc) return done(rc);
          e = cudaEventRecord(ev[k], side);
          if (e != cudaSuccess) return done(cuda_fail(e, "prefill stream join"));
          built_next = true;
        }
      }
      cudaError_t e = lod::launch_prefill_tc_wave(a, maps, pmaps, nsm, st);
      if (e != cudaSuccess) return done(cuda_fail(e, "prefill launch"));
      if (built_next) {
        e = cudaStreamWaitEvent(st, ev[k], 0);
        if (e != cudaSuccess) return done(cuda_fail(e, "prefill stream join"));
      }
    }
    g_err[0] = 0;
    return done(LOD_OK);
  }
  // per-chunk path: 1) the index of every chunk completed inside the query
  // range (a pure function of K/V), 2) attention per query chunk
  if (c1 > c0) {
    rc = do_build(p, K, V, kv_strides, c0, c1, index, ws, st);
    if (rc) return rc;
  }
  // 2) attention, one launch pair per query chunk
  lod::AttendArgs a;
  fill_attend(a, p, s, K, V, kv_strides, index, ws);
  a.q = q;
  a.q_host = q_host;
  a.Tq = Tq;
  a.q_begin = q_begin;
  a.seq_lens = nullptr;
  a.out = out;
  a.lse = lse;
  a.sel_groups = sel_groups;
  a.sel_pages = sel_pages;
  lod::TcMaps maps;
  if (s.tc) {
    rc = make_tc_maps(p, K, V, kv_strides, index, &maps);
    if (rc) return rc;
  }
  const int64_t nw = p->window / p->chunk;
  for (int64_t lo = 0; lo < Tq; lo += p->chunk) {
    const int64_t hi = lo + p->chunk < Tq ? lo + p->chunk : Tq;
    const int64_t bt = (q_begin + lo) / p->chunk;
    const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
    a.pos_lo = lo;
    a.pos_hi = hi;
    a.units = (int64_t)p->B * p->Hkv * cdiv(hi - lo, s.NP);
    const int want = split_for(p, s.tc, a.units, wb * p->clusters + p->window);
    a.nsplit = want < s.nsplit ? want : s.nsplit;
    // part/cand/gsc keep the worst-case layout of fill_attend; a chunk uses a prefix
    cudaError_t e = lod::launch_attend(a, p->dtype, p->d, s.NQ, s.tc ? &maps : nullptr, st);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  }
  g_err[0] = 0;
  return LOD_OK;
}

int32_t lod_get_status(void* ws, lod_stream_t stream, uint32_t* status) {
  if (!ws || !status) return fail(LOD_EINVAL, "ws and status must be non-NULL");
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  *status = v;
  g_err[0] = 0;
  return v ? LOD_EDEVICE : LOD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// lod_decode_noalloc: lod_decode without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc at all: an inference engine whose
// memory pool owns every device allocation, a runtime that must not allocate
// while a CUDA graph or a latency-critical step is being recorded, or a
// plugin host that gives its kernels only their input and output buffers.
// For them this entry point keeps the decode scratch (split partial states,
// group scores and the status word) in a fixed array compiled into the
// library.  The array is `static __device__`, so each GPU that loads this
// library holds its kLodNoallocScratchBytes until the process exits.  Host
// code cannot use the array's name as an address; the device address is
// looked up with cudaGetSymbolAddress, with that device current, on the
// first call made on that device (and again whenever the device's current
// context has changed since, as after cudaDeviceReset).
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kLodNoallocScratchBytes = LOD_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kLodNoallocScratchBytes];

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in, and the address.
// A context that is destroyed and created again (cudaDeviceReset, or a
// driver-API context switch) maps the array at a new address, so the cached
// one is used only while the device's current context is the same.
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};
std::mutex g_noalloc_mu;

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

// The calling thread's current context (null when none is current yet).
int32_t current_context(CUcontext* ctx) {
  std::call_once(g_ctx_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  });
  if (!g_ctx_current) return fail(LOD_ECUDA, "cuCtxGetCurrent is not available from the driver");
  if (g_ctx_current(ctx) != CUDA_SUCCESS) return fail(LOD_ECUDA, "cuCtxGetCurrent failed");
  return LOD_OK;
}

// Device address of the current device's copy of the scratch array, looked
// up on the first call made in the device's current context.
int32_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LOD_EUNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  CUcontext ctx = nullptr;
  int32_t rc = current_context(&ctx);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (ctx == nullptr || ctx != g_noalloc_ctx[dev] || g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    rc = current_context(&ctx);  // the lookup made the device's primary context current if none was
    if (rc) return rc;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return LOD_OK;
}

}  // namespace

extern "C" int32_t lod_decode_noalloc(const lod_params* p, const void* q, const void* K, const void* V,
                                      const int64_t kv_strides[3], const int64_t* seq_lens,
                                      const lod_index* index, void* out, float* lse, int32_t* sel_groups,
                                      int32_t* sel_pages, uint32_t* status, lod_stream_t stream) {
  int32_t rc = validate(p);
  if (!rc) rc = validate_kv(p, K, V, kv_strides);
  if (!rc) rc = validate_index(p, index);
  if (rc) return rc;
  if (!q || !out || !seq_lens) return fail(LOD_EINVAL, "q, out and seq_lens must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(LOD_EINVAL, "q and out must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(status) & 3u) return fail(LOD_EINVAL, "status must be 4-byte aligned");
  const AttendShape s = decode_shape(p);
  const size_t need = attend_ws_bytes(p, s);
  if (need > kLodNoallocScratchBytes)
    return fail(LOD_EINVAL,
                "decode scratch of %zu bytes exceeds the built-in %zu-byte array of lod_decode_noalloc "
                "(fewer sequences, KV heads or a smaller Tmax fit; otherwise use lod_decode)",
                need, kLodNoallocScratchBytes);
  int q_host = 0;
  rc = check_visible(q, "q", &q_host);
  if (!rc) rc = check_visible_all({{out, "out"}, {seq_lens, "seq_lens"}, {lse, "lse"},
                                   {sel_groups, "sel_groups"}, {sel_pages, "sel_pages"}, {status, "status"}});
  if (rc) return rc;
  void* ws = nullptr;
  rc = noalloc_scratch(&ws);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // The partial states and group scores are fully rewritten by every call; only
  // the status word must start from zero when no caller word is given.
  if (!status) {
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the no-alloc status word");
  }
  lod::AttendArgs a;
  fill_attend(a, p, s, K, V, kv_strides, index, ws);
  if (status) a.status = status;
  a.q = q;
  a.q_host = q_host;
  a.Tq = 1;
  a.q_begin = 0;
  a.seq_lens = seq_lens;
  a.pos_lo = 0;
  a.pos_hi = 1;
  a.out = out;
  a.lse = lse;
  a.sel_groups = sel_groups;
  a.sel_pages = sel_pages;
  lod::TcMaps maps;
  if (s.tc) {
    rc = make_tc_maps(p, K, V, kv_strides, index, &maps);
    if (rc) return rc;
  }
  cudaError_t e = lod::launch_attend(a, p->dtype, p->d, s.NQ, s.tc ? &maps : nullptr, st);
  if (e != cudaSuccess) return cuda_fail(e, "no-alloc decode launch");
  g_err[0] = 0;
  return LOD_OK;
}
