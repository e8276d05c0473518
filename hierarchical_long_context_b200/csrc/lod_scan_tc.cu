// lod_scan_tc.cu -- the coarse scan of LoD attention on tcgen05 tensor cores
// (bf16 caches, d = 128).
//
// "Level of Detail Attention", section "How It Works": every visible group
// summary (mean key, mean value, ln count) and every window token of one
// (sequence, KV head) enters one online softmax for each of the unit's query
// rows, and each split keeps its best `top_groups` groups per query row for
// the groups to open.  A unit's rows are cut into tiles of 128; a CTA streams a
// contiguous run of tiles through a warp-specialised pipeline:
//
//   warp 0     producer: TMA copies of the K and V tiles (two 64-column boxes
//              each, 128B swizzle) into a three-stage ring, plus cp.async
//              copies of the group counts; group tiles come from the summary
//              arrays, window tiles from the KV cache.
//   warp 1     one thread issues the MMAs:
//                S[128 rows x 16] = K_tile . Q^T   into one of two TMEM
//                                                  score buffers
//                O[128 dims x 16] += V_tile^T . P^T accumulated in TMEM over
//                                                  all tiles of the split
//              MMA 1 of tile i+1 runs while the softmax warps work on tile i.
//   warps 2-5  softmax, one thread per tile row (warp w reads TMEM lane
//              quadrant w % 4): weights p = exp(score + ln count - m) with a
//              reference max m per query row that only moves when a logit
//              exceeds it by more than kTau (then the four warps agree on the
//              tile max and rescale O in TMEM); p goes to shared memory as the
//              bf16 B operand of MMA 2; per-thread partial sums; each
//              group tile's scores, transposed, go to a double-buffered
//              shared-memory slot for the selection warps.
//   warps 6-9  each query row's best `top_groups` groups of the split: 16
//              threads per query row each keep, in registers, the best G of
//              every 16th group (score, then smaller id); a group enters a
//              list only if it beats the list's G-th best and the row's
//              bound (the largest G-th best of the 16 lists: G groups reach
//              it).  At the end the 16 lists are merged, G rounds of a
//              16-lane maximum, into the split's G best, from which the
//              refine kernel picks the groups to open.
//
// The partial state (m, l, acc[d]) is written in the same layout as the
// CUDA-core scan, so the refine kernel is shared.  acc and l are relative to
// the reference max m (every weight is at most e^kTau).
#include <cudaTypedefs.h>

#include "lod_internal.cuh"
#include "lod_tc.cuh"

namespace lod {

namespace {

constexpr int D = 128;
constexpr int N = 16;            // MMA N: the unit's query rows (<= 8), zero padded
constexpr int TROWS = 128;       // rows per tile: MMA 1's M, MMA 2's K
constexpr int kStages = 3;
constexpr int kThreads = 320;    // warp 0 copies, warp 1 issues MMAs, warps 2-5 softmax, 6-9 selection
constexpr int kSoftThreads = 128;
constexpr int kBarSoft = 1;      // named barrier of the softmax warps
constexpr uint32_t kTileBytes = TROWS * D * 2;  // one operand tile: 32 KB
constexpr float kTau = 8.f;      // weights reach at most e^kTau before m moves
constexpr uint32_t kTmemCols = 64;  // S buffers in columns [0, 32), O in [32, 48)
constexpr uint32_t kColO = 32;
constexpr int kTS = TROWS + 16;  // row stride of the transposed group scores (floats)

struct TcSmem {
  static constexpr size_t off_K = 0;                                       // [stages][2][128][128 B]
  static constexpr size_t off_V = off_K + (size_t)kStages * kTileBytes;
  static constexpr size_t off_Q = off_V + (size_t)kStages * kTileBytes;    // [2][16][128 B]
  static constexpr size_t off_P = off_Q + 2 * N * 128;                     // [2 bufs][2][16][128 B]
  static constexpr size_t off_cnt = off_P + 4 * N * 128;                   // int [stages][128]
  static constexpr size_t off_red = off_cnt + sizeof(int) * kStages * TROWS;  // float [4][8]
  static constexpr size_t off_flag = off_red + sizeof(float) * 4 * 8;         // int abort flag
  static constexpr size_t off_sT = off_flag + 16;                      // float [2][8][kTS] group scores
  static constexpr size_t off_sM = off_sT + sizeof(float) * 2 * 8 * kTS;  // int [2][128] their gMeta words
  static constexpr int kBars = 2 * kStages + 4 * 2 + 1 + 4;
  static constexpr size_t off_bar = (off_sM + 4 * 2 * TROWS + 7) & ~size_t(7);
  static constexpr size_t off_tmem = off_bar + 8 * kBars;
  static constexpr size_t bytes = off_tmem + 16 + 1024;  // + alignment slack
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Insert (v, id, meta) into the descending list (s, ix, mt) of GM entries:
// every entry from the first one v beats moves down by one place (ties keep
// the earlier entry, which has the smaller id).  A list of G < GM entries
// occupies the last G slots below GM - G sentinels of +inf, so that its G-th
// best is always s[GM - 1]; selects only, so the list stays in registers.
template <int GM>
__device__ __forceinline__ void list_insert(float (&s)[GM], int (&ix)[GM], int (&mt)[GM], float v, int id, int meta) {
  bool act = false;
  float cs = v;
  int ci = id, cm = meta;
#pragma unroll
  for (int k = 0; k < GM; ++k) {
    act = act || (v > s[k]);
    const float ns = act ? cs : s[k];
    const int ni = act ? ci : ix[k];
    const int nm = act ? cm : mt[k];
    cs = act ? s[k] : cs;
    ci = act ? ix[k] : ci;
    cm = act ? mt[k] : cm;
    s[k] = ns;
    ix[k] = ni;
    mt[k] = nm;
  }
}

template <int NQ, int GM>
__global__ void __launch_bounds__(kThreads, 1)
    scan_tc_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ AttendArgs a) {
  static_assert(NQ <= 8, "query rows per unit");
  static_assert(N * (D / 8) % kSoftThreads == 0, "query pieces per softmax thread");
  const int64_t u = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  unsigned char* Kring = sm + TcSmem::off_K;
  unsigned char* Vring = sm + TcSmem::off_V;
  unsigned char* Qs = sm + TcSmem::off_Q;
  unsigned char* Ps = sm + TcSmem::off_P;
  int* cnt_s = reinterpret_cast<int*>(sm + TcSmem::off_cnt);
  float* sT = reinterpret_cast<float*>(sm + TcSmem::off_sT);
  int* sM = reinterpret_cast<int*>(sm + TcSmem::off_sM);
  float* red = reinterpret_cast<float*>(sm + TcSmem::off_red);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + TcSmem::off_flag);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + TcSmem::off_bar);  // K/V tile + counts landed
  uint64_t* empty = full + kStages;                                     // ring slot free again
  uint64_t* s_full = empty + kStages;                                   // scores of tile i in TMEM
  uint64_t* s_free = s_full + 2;                                        // score buffer read out
  uint64_t* p_full = s_free + 2;                                        // weights of tile i written
  uint64_t* o_done = p_full + 2;                                        // MMA 2 of tile i complete
  uint64_t* fin = o_done + 2;                                           // every MMA complete
  uint64_t* sel_full = fin + 1;                                         // a group tile's scores transposed
  uint64_t* sel_free = sel_full + 2;                                    // the selection has read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + TcSmem::off_tmem);

  // ---- unit (decode: (b, kvh); prefill: (b, kvh, position block))
  int b, kvh;
  int64_t blk = 0;
  if (a.seq_lens) {
    b = (int)(u / a.Hkv);
    kvh = (int)(u % a.Hkv);
  } else {
    const int64_t nblk = (a.pos_hi - a.pos_lo + a.NP - 1) / a.NP;
    b = (int)(u / (a.Hkv * nblk));
    kvh = (int)((u / nblk) % a.Hkv);
    blk = u % nblk;
  }

  // ---- set-up that reads no input, done while the preceding kernel drains:
  // barriers and tensor maps (warp 0), TMEM (warp 1), zeroed weights and the
  // query rows brought into L2 (softmax warps)
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1 + 32);  // the producer's expect_tx + 32 cp.async arrivals
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(fin, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sel_full[i], 4);
      mbar_init(&sel_free[i], 4);
    }
    *abort_s = 0;
    fence_mbar_init();
    tc::prefetch_tensormap(&maps.gK);
    tc::prefetch_tensormap(&maps.gV);
    tc::prefetch_tensormap(&maps.K);
    tc::prefetch_tensormap(&maps.V);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, kTmemCols);
  if (warp >= 2 && warp < 6) {
    const int t = tid - 64;
    for (int c2 = t; c2 < 4 * N * 128 / 16; c2 += kSoftThreads)
      reinterpret_cast<uint4*>(Ps)[c2] = make_uint4(0, 0, 0, 0);
    // (an L2 prefetch has no effect on what a later load returns)
    const int r = t >> 1;
    const int64_t pi = a.seq_lens ? 0 : a.pos_lo + blk * a.NP + r / a.g;
    if (r < NQ && (a.seq_lens ? r < a.g : (r < a.g * a.NP && pi < a.pos_hi))) {
      const int hq = kvh * a.g + (r % a.g);
      prefetch_l2(static_cast<const __nv_bfloat16*>(a.q) + (((int64_t)b * a.Hq + hq) * a.Tq + pi) * D + (t & 1) * 64);
    }
  }

  // query piece i of this softmax thread (16 bytes; zero for a missing row)
  constexpr int kQPer = N * (D / 8) / kSoftThreads;  // 16-byte pieces per softmax thread
  auto load_q = [&](int i) {
    const int c2 = (tid - 64) + i * kSoftThreads;
    const int r = c2 / (D / 8), c = c2 % (D / 8);
    const int64_t pi = a.seq_lens ? 0 : a.pos_lo + blk * a.NP + r / a.g;
    const bool row = r < NQ && (a.seq_lens ? r < a.g : (r < a.g * a.NP && pi < a.pos_hi));
    if (!row) return make_uint4(0, 0, 0, 0);
    const int hq = kvh * a.g + (r % a.g);
    return __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                 (((int64_t)b * a.Hq + hq) * a.Tq + pi) * D) + c);
  };
  // q in host memory was written by the host before the call was enqueued
  // (the entry points' contract), so its loads over the host link go out
  // before the dependency wait, overlapping the preceding kernel (which rows
  // exist does not depend on the sequence length; rows of an invalid
  // sequence are zeroed below); q in device memory is read after the wait
  uint4 qv[kQPer];
#pragma unroll
  for (int i = 0; i < kQPer; ++i) qv[i] = make_uint4(0, 0, 0, 0);
  if (warp >= 2 && warp < 6 && a.q_host) {
#pragma unroll
    for (int i = 0; i < kQPer; ++i) qv[i] = load_q(i);
  }

  // launched as a programmatic dependent: device inputs are read only after
  // the preceding kernel has completed; the refine kernel may launch right away
  // (it waits for this grid's completion before reading what it writes)
  pdl_wait();
  pdl_launch_dependents();

  int64_t t_row[NQ];
  bool ok[NQ];
  int64_t t_max = -1;
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    if (a.seq_lens) {
      const int64_t L = a.seq_lens[b];
      ok[r] = (r < a.g) && L >= 1 && L <= a.Tmax;
      t_row[r] = L - 1;
    } else {
      const int64_t pi = a.pos_lo + blk * a.NP + r / a.g;
      ok[r] = (r < a.g * a.NP) && pi < a.pos_hi;
      t_row[r] = a.q_begin + pi;
    }
    if (ok[r] && t_row[r] > t_max) t_max = t_row[r];
  }
  if (a.seq_lens && t_max < 0 && s == 0 && tid == 0) set_status(a.status, LOD_ST_BAD_SEQLEN);

  // ---- this split's tiles: group tiles [0, gt), then window tiles (the
  // sinks are exact tokens added by the refine kernel)
  const int64_t unit_kv = (int64_t)b * a.Hkv + kvh;
  int64_t G_vis = 0, ws = 0, gt = 0, t0 = 0, t1 = 0;
  if (t_max >= 0) {
    const int64_t bt = t_max / kChunk;
    const int64_t nw = a.window / kChunk;
    const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
    ws = wb * kChunk;
    G_vis = wb * a.k;
    const int64_t wn = t_max - ws + 1;
    gt = (G_vis + TROWS - 1) / TROWS;
    const int64_t total = gt + (wn + TROWS - 1) / TROWS;
    const int64_t per = (total + a.nsplit - 1) / a.nsplit;
    t0 = s * per < total ? s * per : total;
    t1 = t0 + per < total ? t0 + per : total;
  }
  const int ntile = (int)(t1 - t0);
  const int64_t grow0 = unit_kv * a.Cmax * a.k;  // this unit's first summary row
  const int32_t* gM = a.gMeta + grow0;  // size | page range per group

  // producer (warp 0, all lanes): tile t0 + i into ring slot i % kStages;
  // the tiles are read once per call (evict-first in L2)
  const uint64_t l2pol = l2_policy_evict_first();
  auto issue_tile = [&](int i) {
    const int st = i % kStages;
    const int64_t tile = t0 + i;
    unsigned char* kd = Kring + (size_t)st * kTileBytes;
    unsigned char* vd = Vring + (size_t)st * kTileBytes;
    if (lane == 0) {
      mbar_arrive_expect(&full[st], 2u * kTileBytes);
      if (tile < gt) {
        const int row = (int)(grow0 + tile * TROWS);
        tc::tma_load_2d(kd, &maps.gK, 0, row, &full[st], l2pol);
        tc::tma_load_2d(kd + kTileBytes / 2, &maps.gK, 64, row, &full[st], l2pol);
        tc::tma_load_2d(vd, &maps.gV, 0, row, &full[st], l2pol);
        tc::tma_load_2d(vd + kTileBytes / 2, &maps.gV, 64, row, &full[st], l2pol);
      } else {
        const int pos = (int)(ws + (tile - gt) * TROWS);
        tc::tma_load_4d(kd, &maps.K, 0, pos, kvh, b, &full[st], l2pol);
        tc::tma_load_4d(kd + kTileBytes / 2, &maps.K, 64, pos, kvh, b, &full[st], l2pol);
        tc::tma_load_4d(vd, &maps.V, 0, pos, kvh, b, &full[st], l2pol);
        tc::tma_load_4d(vd + kTileBytes / 2, &maps.V, 64, pos, kvh, b, &full[st], l2pol);
      }
    }
    if (tile < gt) {  // the tile's groups' size and page range (zero past the visible ones)
#pragma unroll
      for (int k4 = 0; k4 < TROWS / 32; ++k4) {
        const int r = lane + 32 * k4;
        const int64_t gid = tile * TROWS + r;
        const bool v = gid < G_vis;
        cp_async4_zfill(cnt_s + st * TROWS + r, v ? gM + gid : gM, v);
      }
    }
    cp_async_mbar_arrive_noinc(&full[st]);
  };

  // ---- the first ring stages (warp 0) and the query operand (softmax warps)
  if (warp == 0) {
    __syncwarp();
    for (int i = 0; i < kStages && i < ntile; ++i) issue_tile(i);
  }
  if (warp >= 2 && warp < 6) {
    const int t = tid - 64;
#pragma unroll
    for (int i = 0; i < kQPer; ++i) {
      const int c2 = t + i * kSoftThreads;
      const int r = c2 / (D / 8), c = c2 % (D / 8);
      bool okr = false;
#pragma unroll
      for (int x = 0; x < NQ; ++x)
        if (x == r) okr = ok[x];
      if (okr && !a.q_host) qv[i] = load_q(i);
      const uint4 v = okr ? qv[i] : make_uint4(0, 0, 0, 0);
      const uint32_t off = (uint32_t)((c >> 3) * (N * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
      *reinterpret_cast<uint4*>(Qs + off) = v;
    }
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // bounded wait that also gives up once another role has given up
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_s) return false;
    if (mbar_wait(bar, parity, a.status)) return true;
    *abort_s = 1;
    return false;
  };

  if (warp == 0) {
    // ================================================================ producer
    int issued = ntile < kStages ? ntile : kStages;  // issued during the set-up
    for (int i = kStages; i < ntile; ++i) {
      if (!wait(&empty[i % kStages], (uint32_t)(i / kStages - 1) & 1u)) break;
      issue_tile(i);
      ++issued;
    }
    cp_async_wait_all();
    if (*abort_s && lane == 0) {  // let the copies still in flight land before the CTA ends
      for (int i = issued - 1; i >= 0 && i >= issued - kStages; --i)
        (void)mbar_wait(&full[i % kStages], (uint32_t)(i / kStages) & 1u, a.status);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issue
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16(TROWS, N, false, false);
      const uint32_t id2 = tc::idesc_bf16(D, N, true, false);
      auto mma2 = [&](int t) -> bool {  // O += V_t^T . P_t^T
        if (!wait(&p_full[t & 1], (uint32_t)(t >> 1) & 1u)) return false;
        tc::fence_after_sync();
        const int st = t % kStages;
        const uint32_t vbase = smem_u32(Vring + (size_t)st * kTileBytes);
        const uint32_t pbase = smem_u32(Ps + (size_t)(t & 1) * (2 * N * 128));
#pragma unroll
        for (int kk = 0; kk < TROWS / 16; ++kk) {
          const uint64_t ad = tc::desc_mnmajor_sw128(vbase + kk * 2048, kTileBytes / 2);
          const uint64_t bd = tc::desc_kmajor_sw128(pbase + (kk / 4) * (N * 128) + (kk % 4) * 32);
          tc::mma_bf16(tmem + kColO, ad, bd, id2, t > 0 || kk > 0);
        }
        tc::mma_commit(&o_done[t & 1]);
        tc::mma_commit(&empty[st]);
        return true;
      };
      bool go = true, any_mma = false;
      for (int i = 0; i < ntile && go; ++i) {
        const int st = i % kStages;
        if (!wait(&full[st], (uint32_t)(i / kStages) & 1u)) break;
        if (i >= 2 && !wait(&s_free[i & 1], (uint32_t)((i - 2) >> 1) & 1u)) break;
        tc::fence_after_sync();
        // S_i = K_i . Q^T
        const uint32_t kbase = smem_u32(Kring + (size_t)st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = tc::desc_kmajor_sw128(kbase + (kk / 4) * (kTileBytes / 2) + (kk % 4) * 32);
          const uint64_t bd = tc::desc_kmajor_sw128(smem_u32(Qs) + (kk / 4) * (N * 128) + (kk % 4) * 32);
          tc::mma_bf16(tmem + (uint32_t)(i & 1) * N, ad, bd, id1, kk > 0);
        }
        tc::mma_commit(&s_full[i & 1]);
        any_mma = true;
        if (i >= 1) go = mma2(i - 1);
        if (go && i == ntile - 1) go = mma2(i);
      }
      if (any_mma) {  // every MMA done before TMEM is released
        tc::mma_commit(fin);
        (void)mbar_wait(fin, 0, a.status);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ================================================================ softmax
    const int q = warp & 3, wq = warp - 2;
    const int r = 32 * q + lane;  // tile row of this thread, and O's dim at the end
    const uint32_t tlane = (uint32_t)(32 * q) << 16;
    float m[NQ], l[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      m[j] = -INFINITY;
      l[j] = 0.f;
    }
    bool alive = true;
    for (int i = 0; i < ntile; ++i) {
      const int st = i % kStages, buf = i & 1;
      const int64_t tile = t0 + i;
      const bool is_group = tile < gt;
      const int64_t r0 = is_group ? tile * TROWS : ws + (tile - gt) * TROWS;  // first row id / position
      // (a failed wait is carried to the next softmax barrier, where the four
      // warps leave the loop together)
      alive = __all_sync(0xffffffffu, wait(&full[st], (uint32_t)(i / kStages) & 1u) &&
                                          wait(&s_full[buf], (uint32_t)(i >> 1) & 1u));
      float sv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) sv[j] = 0.f;
      if (alive) {
        tc::fence_after_sync();
        tc::tmem_ld8(tmem + tlane + (uint32_t)buf * N, sv);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[buf]);
      }
      // ln count of row r; -inf: the row is in no query row's softmax
      float lc;
      int meta = 0;
      if (is_group) {
        meta = cnt_s[st * TROWS + r];
        const int c = meta & 0xffff;
        lc = (c > 0 && c <= kChunk) ? __logf((float)c) : -INFINITY;
        if (c > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
      } else {
        lc = r0 + r <= t_max ? 0.f : -INFINITY;
      }
      float sc[NQ], lg[NQ];
      bool need = false;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        sc[j] = sv[j] * a.scale;
        const bool live = ok[j] && lc != -INFINITY && (is_group || r0 + r <= t_row[j]);
        lg[j] = live ? sc[j] + lc : -INFINITY;
        need |= lg[j] > m[j] + kTau;
      }
      if (bar_red_or(kBarSoft, kSoftThreads, need || !alive)) {
        if (bar_red_or(kBarSoft, kSoftThreads, !alive)) {
          alive = false;
          break;
        }
        // the reference max moves to the tile max; O and the sums follow
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
          const float wm = warp_max(lg[j]);
          if (lane == 0) red[wq * 8 + j] = wm;
        }
        bar_named_sync(kBarSoft, kSoftThreads);
        float corr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) corr[j] = 1.f;
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
          const float tm = fmaxf(fmaxf(red[j], red[8 + j]), fmaxf(red[16 + j], red[24 + j]));
          const float mn = fmaxf(m[j], tm);
          corr[j] = m[j] == -INFINITY ? 0.f : __expf(m[j] - mn);
          m[j] = mn;
          l[j] *= corr[j];
        }
        if (i > 0) alive = __all_sync(0xffffffffu, wait(&o_done[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u));
        if (i > 0 && alive) {
          tc::fence_after_sync();
          float ov[8];
          tc::tmem_ld8(tmem + tlane + kColO, ov);
#pragma unroll
          for (int j = 0; j < 8; ++j) ov[j] *= corr[j];
          tc::tmem_st8(tmem + tlane + kColO, ov);
        }
      }
      // weights into the B operand of MMA 2 (its buffer is free once MMA 2 of tile i-2 is done)
      if (i >= 2 && !wait(&o_done[buf], (uint32_t)((i - 2) >> 1) & 1u)) alive = false;
      unsigned char* Pb = Ps + (size_t)buf * (2 * N * 128);
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const float p = lg[j] == -INFINITY ? 0.f : __expf(lg[j] - m[j]);
        l[j] += p;
        *reinterpret_cast<__nv_bfloat16*>(Pb + tc::sw128_offset(j, r, N)) = __float2bfloat16_rn(p);
      }
      // a row in no softmax must not bring NaN/Inf into MMA 2
      if (lc == -INFINITY) {
        unsigned char* vd = Vring + (size_t)st * kTileBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(vd + h * (kTileBytes / 2) + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[buf]);
      // the group tile's scores, transposed (-inf: not in the row's
      // softmax), and gMeta words for the selection warps (group tiles come
      // first in a split: group tile i is tile i)
      if (is_group) {
        const int sb = i & 1;
        if (i >= 2 && !wait(&sel_free[sb], (uint32_t)((i - 2) >> 1) & 1u)) alive = false;
        if (alive) {
          const bool vg = r0 + r < G_vis;
#pragma unroll
          for (int j = 0; j < NQ; ++j) sT[(sb * 8 + j) * kTS + r] = (vg && lg[j] != -INFINITY) ? sc[j] : -INFINITY;
          sM[sb * TROWS + r] = meta;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sel_full[sb]);
      }
    }
    // ---------------------------------------------------------------- epilogue
    alive = !bar_red_or(kBarSoft, kSoftThreads, !alive);
    // O (this thread's dim r, query rows 0..7), once the last MMA 2 is done
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (alive && ntile > 0) {
      alive = __all_sync(0xffffffffu, wait(&o_done[(ntile - 1) & 1], (uint32_t)((ntile - 1) >> 1) & 1u));
      if (alive) {
        tc::fence_after_sync();
        tc::tmem_ld8(tmem + tlane + kColO, acc);
      }
    }
    alive = !bar_red_or(kBarSoft, kSoftThreads, !alive);
    // sums over the 128 rows
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const float lw = warp_sum(l[j]);
      if (lane == 0) red[wq * 8 + j] = lw;
    }
    bar_named_sync(kBarSoft, kSoftThreads);
    float* part = a.part + ((u * a.nsplit + s) * NQ) * (int64_t)(D + 2);
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      part[j * (D + 2) + 2 + r] = alive ? acc[j] : 0.f;
      if (wq == 0 && lane == j) {
        part[j * (D + 2) + 0] = alive ? m[j] : -INFINITY;
        part[j * (D + 2) + 1] = alive ? red[j] + red[8 + j] + red[16 + j] + red[24 + j] : 0.f;
      }
    }
  } else {
    // ================================================================ selection
    // this thread keeps the best G of query row jr's groups c, c + 16, c + 32,
    // ... of every group tile (t = 16 jr + c); rows >= NQ keep empty lists
    const int t = tid - 192, jr = t >> 4, cls = t & 15;
    const int G = a.G;
    float ls[GM];
    int li[GM], lm[GM];
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      ls[k] = k < GM - G ? INFINITY : -INFINITY;
      li[k] = -1;
      lm[k] = 0;
    }
    float bnd = -INFINITY;  // the largest G-th best of the row's 16 lists
    bool alive = true;
    const int ngt = (int)((t1 < gt ? t1 : gt) - t0);  // group tiles of this split
    for (int i = 0; i < ngt; ++i) {
      const int sb = i & 1;
      alive = __all_sync(0xffffffffu, wait(&sel_full[sb], (uint32_t)(i >> 1) & 1u));
      if (!alive) break;
      // a group enters a list if it beats both the list's G-th best and the
      // row's bound (the tile's groups all have larger ids than those behind
      // the bound, so a tie with it loses)
      if (jr < NQ) {
        const int64_t r0 = (t0 + i) * TROWS;
        float v8[TROWS / 16];
        unsigned cm = 0;  // this lane's candidates (bit e8: group cls + 16 e8)
        const float th = fmaxf(ls[GM - 1], bnd);
#pragma unroll
        for (int e8 = 0; e8 < TROWS / 16; ++e8) {
          v8[e8] = sT[(sb * 8 + jr) * kTS + cls + 16 * e8];
          cm |= (v8[e8] > th ? 1u : 0u) << e8;
        }
        while (cm) {  // in id order; each must still beat the list's G-th best
          const int e8 = __ffs(cm) - 1;
          cm &= cm - 1;
          float v = v8[0];
#pragma unroll
          for (int x = 1; x < TROWS / 16; ++x) v = x == e8 ? v8[x] : v;
          const int e = cls + 16 * e8;
          if (v > fmaxf(ls[GM - 1], bnd)) list_insert<GM>(ls, li, lm, v, (int)(r0 + e), sM[sb * TROWS + e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sel_free[sb]);
      float kb = ls[GM - 1];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) kb = fmaxf(kb, __shfl_xor_sync(0xffffffffu, kb, o));
      bnd = fmaxf(bnd, kb);
    }
    // the split's best G of row jr: G rounds in which each of the row's 16
    // lists offers its best entry not yet taken and the largest key wins
    // (lanes of both rows of a warp run every round: the shuffles take the
    // whole warp)
    SplitCand* co = a.cand + ((u * a.nsplit + s) * NQ + (jr < NQ ? jr : 0)) * G;
    int h = GM - G, kept = 0;
    for (int k = 0; k < G; ++k) {
      float hs = -INFINITY;
      int hid = -1, hm = 0;
#pragma unroll
      for (int x = 0; x < GM; ++x)
        if (x == h) {
          hs = ls[x];
          hid = li[x];
          hm = lm[x];
        }
      const uint64_t mine = (alive && jr < NQ && h < GM && hs != -INFINITY) ? group_key(hs, hid) : 0ull;
      uint64_t best = mine;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const uint64_t x = __shfl_xor_sync(0xffffffffu, best, o);
        best = x > best ? x : best;
      }
      if (best != 0ull) {
        kept = k + 1;
        if (mine == best) {  // one list holds it: group ids are distinct
          SplitCand c;
          c.s = hs;
          c.id = hid;
          c.meta = hm;
          c.pad = 0;
          co[k] = c;
          ++h;
        }
      }
    }
    if (jr < NQ && cls < G && cls >= kept) {
      SplitCand c;
      c.s = -INFINITY;
      c.id = -1;
      c.meta = 0;
      c.pad = 0;
      co[cls] = c;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

template <int NQ>
cudaError_t launch_nq(const AttendArgs& a, const TcMaps& maps, cudaStream_t stream) {
  // registers for the group lists: G <= 8 or G <= 16 entries
  auto kern = a.G <= 8 ? scan_tc_kernel<NQ, 8> : scan_tc_kernel<NQ, 16>;
  const size_t smem = TcSmem::bytes;
  cudaError_t e = a.G <= 8 ? set_smem_once<scan_tc_kernel<NQ, 8>>(smem) : set_smem_once<scan_tc_kernel<NQ, 16>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)a.units, (unsigned)a.nsplit), dim3(kThreads), smem, stream, maps, a);
}

}  // namespace

cudaError_t launch_scan_tc(const AttendArgs& a, const TcMaps& maps, int NQ, cudaStream_t stream) {
  switch (NQ) {
    case 1: return launch_nq<1>(a, maps, stream);
    case 2: return launch_nq<2>(a, maps, stream);
    case 4: return launch_nq<4>(a, maps, stream);
    case 8: return launch_nq<8>(a, maps, stream);
    default: return cudaErrorInvalidValue;
  }
}

size_t scan_tc_smem_bytes() { return TcSmem::bytes; }

}  // namespace lod
