// lod_scan_tc.cu -- the group/window scan of LoD attention on the sm_100
// tensor cores (bf16, d = 128).
//
// Same job as the CUDA-core scan in lod_attend.cu ("Level of Detail
// Attention", How It Works, paragraphs 2-3): every visible group summary
// (mean key, mean value, ln count) and every window token of one (sequence,
// KV head) enters an online softmax for each of the unit's query rows, and
// the best `top_groups` groups by score are kept as candidates.  The unit's
// rows are cut into tiles of 128; a CTA streams a contiguous run of tiles:
//
//   TMA     K and V tiles (two 64-column boxes each, 128B swizzle) into a
//           three-stage ring; group tiles come from the summary arrays, window
//           tiles from the KV cache.
//   MMA 1   S[128 rows x 16] = K_tile . Q^T   (tcgen05, fp32 in TMEM); the
//           unit's <= 16 query rows are the N dimension (zero padded).
//   CUDA    16 warps read the scores from TMEM (warp w: lane quadrant w % 4,
//           columns 4 (w / 4) .. +3); warp j then owns query row j: the tile
//           max, the new running max, the weights
//           p = exp(score + ln count - max) (written to shared memory as the
//           bf16 B operand of MMA 2), the running sum, and the top-KG groups.
//   MMA 2   O[128 dims x 16] = V_tile^T . P^T  (fresh TMEM block per tile);
//           each thread folds its 4 (dim, query row) entries into
//           acc = acc * corr[row] + O.
//
// The partial state (max, sum, acc[d]) and the candidates are written in the
// same layout as the CUDA-core scan, so the refine kernel is shared.
#include <cudaTypedefs.h>

#include "lod_internal.cuh"
#include "lod_tc.cuh"

namespace lod {

namespace {

constexpr int D = 128;
constexpr int N = 16;           // MMA N: query rows per unit, padded
constexpr int TROWS = 128;      // rows per tile (MMA M)
constexpr int kTcStages = 3;
constexpr int kTcThreads = 512;  // 16 warps: 4 TMEM lane quadrants x 4 column groups
constexpr uint32_t kTileBytes = TROWS * D * 2;  // one operand tile: 32 KB

struct TcSmem {
  static constexpr size_t off_K = 0;                                   // [stages][2][128][128 B]
  static constexpr size_t off_V = off_K + (size_t)kTcStages * kTileBytes;
  static constexpr size_t off_Q = off_V + (size_t)kTcStages * kTileBytes;  // [2][16][128 B]
  static constexpr size_t off_P = off_Q + 2 * N * 128;                  // [2][16][128 B]
  static constexpr size_t off_S = off_P + 2 * N * 128;                  // float [16][128] scores
  static constexpr size_t off_lnc = off_S + sizeof(float) * N * TROWS;  // float [128]
  static constexpr size_t off_corr = off_lnc + sizeof(float) * TROWS;   // float [16]
  static constexpr size_t off_pmax = off_corr + sizeof(float) * N;      // float [2][16] pair maxima
  static constexpr size_t off_meta = off_pmax + sizeof(float) * 2 * N;  // int [2][128]: count, page range
  static constexpr size_t off_bar = off_meta + sizeof(int) * 2 * TROWS;  // uint64 [kTcStages + 2]
  static constexpr size_t off_tmem = off_bar + 8 * (kTcStages + 2);
  static constexpr size_t bytes = off_tmem + 16 + 1024;  // + alignment slack
};

struct Cand {
  float s;
  int id;
  int pages;
  int cnt;
};

template <int NQ, int KG>
__global__ void __launch_bounds__(kTcThreads, 1)
    scan_tc_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ AttendArgs a) {
  static_assert(NQ <= 8, "query rows per unit (two warps per row)");
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
  float* S_s = reinterpret_cast<float*>(sm + TcSmem::off_S);
  float* lnc_s = reinterpret_cast<float*>(sm + TcSmem::off_lnc);
  float* corr_s = reinterpret_cast<float*>(sm + TcSmem::off_corr);
  float* pmax_s = reinterpret_cast<float*>(sm + TcSmem::off_pmax);
  int* cnt_s = reinterpret_cast<int*>(sm + TcSmem::off_meta);      // group size of row r
  int* pgs_s = cnt_s + TROWS;                                      // page range of row r
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + TcSmem::off_bar);
  uint64_t* bar_s = full + kTcStages;
  uint64_t* bar_o = full + kTcStages + 1;
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

  // ---- this split's tiles: group tiles [0, gt), then window tiles
  const int64_t unit_kv = (int64_t)b * a.Hkv + kvh;
  int64_t G_vis = 0, ws = 0, wn = 0, gt = 0, t0 = 0, t1 = 0;
  if (t_max >= 0) {
    const int64_t bt = t_max / kChunk;
    const int64_t nw = a.window / kChunk;
    const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
    ws = wb * kChunk;
    G_vis = wb * a.k;
    wn = t_max - ws + 1;
    gt = (G_vis + TROWS - 1) / TROWS;
    const int64_t total = gt + (wn + TROWS - 1) / TROWS;
    const int64_t per = (total + a.nsplit - 1) / a.nsplit;
    t0 = s * per < total ? s * per : total;
    t1 = t0 + per < total ? t0 + per : total;
  }
  const int ntile = (int)(t1 - t0);
  const int64_t grow0 = unit_kv * a.Cmax * a.k;  // this unit's first summary row
  const int32_t* gC = a.gCnt + grow0;

  // ---- set-up: barriers, first tiles in flight, TMEM, the query operand
  if (tid == 0) {
    for (int i = 0; i < kTcStages + 2; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int i) {  // by thread 0: tile t0 + i into ring slot i % kTcStages
    const int st = i % kTcStages;
    const int64_t tile = t0 + i;
    unsigned char* kd = Kring + (size_t)st * kTileBytes;
    unsigned char* vd = Vring + (size_t)st * kTileBytes;
    mbar_arrive_expect(&full[st], 2u * kTileBytes);
    if (tile < gt) {
      const int row = (int)(grow0 + tile * TROWS);
      tc::tma_load_2d(kd, &maps.gK, 0, row, &full[st]);
      tc::tma_load_2d(kd + kTileBytes / 2, &maps.gK, 64, row, &full[st]);
      tc::tma_load_2d(vd, &maps.gV, 0, row, &full[st]);
      tc::tma_load_2d(vd + kTileBytes / 2, &maps.gV, 64, row, &full[st]);
    } else {
      const int pos = (int)(ws + (tile - gt) * TROWS);
      tc::tma_load_4d(kd, &maps.K, 0, pos, kvh, b, &full[st]);
      tc::tma_load_4d(kd + kTileBytes / 2, &maps.K, 64, pos, kvh, b, &full[st]);
      tc::tma_load_4d(vd, &maps.V, 0, pos, kvh, b, &full[st]);
      tc::tma_load_4d(vd + kTileBytes / 2, &maps.V, 64, pos, kvh, b, &full[st]);
    }
  };
  if (tid == 0)
    for (int i = 0; i < kTcStages - 1 && i < ntile; ++i) issue(i);
  if (warp == 0) tc::tmem_alloc(tmem_slot, 32);
  // the query rows, 16-byte chunks into the swizzled K-major layout; P zeroed
  if (tid < N * (D / 8)) {
    const int r = tid / (D / 8), c = tid % (D / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    bool okr = false;
#pragma unroll
    for (int x = 0; x < NQ; ++x)
      if (x == r) okr = ok[x];
    if (r < NQ && okr) {
      const int hq = kvh * a.g + (r % a.g);
      const int64_t pi = a.seq_lens ? 0 : a.pos_lo + blk * a.NP + r / a.g;
      v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                (((int64_t)b * a.Hq + hq) * a.Tq + pi) * D) + c);
    }
    const uint32_t off = (uint32_t)((c >> 3) * (N * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
    *reinterpret_cast<uint4*>(Qs + off) = v;
    *reinterpret_cast<uint4*>(Ps + off) = make_uint4(0, 0, 0, 0);
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // running state: query row j is shared by warps j and j + 8, each taking 64
  // rows of every tile; each keeps (m, l) over its rows (m is common to the
  // pair).  Every lane keeps a private sorted top-KG of the group rows it sees
  // (score, id, page range, count); the lists are merged once, at the end.
  float m_run = -INFINITY, l_run = 0.f;
  float ls[KG];
  int lid[KG], lpg[KG], lcn[KG];
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    ls[k] = -INFINITY;
    lid[k] = 0x7fffffff;
    lpg[k] = lcn[k] = 0;
  }
  const int quad = warp & 3, cgrp = warp >> 2;  // TMEM lane quadrant, column group
  // row `tid` (< 128) of the next group tile: count and page range, prefetched
  const int16_t* gP = a.gPage + unit_kv * a.Cmax * (a.k + 1);
  auto fetch_meta = [&](int64_t tile, int& cnt, int& pg) {
    cnt = 0;
    pg = 0;
    if (tile < gt && tid < TROWS && tile * TROWS + tid < G_vis) {
      const int64_t gid = tile * TROWS + tid;
      cnt = gC[gid];
      const int16_t* gp = gP + (gid / a.k) * (a.k + 1) + gid % a.k;
      pg = ((int)(uint16_t)gp[0]) | ((int)(uint16_t)gp[1] << 16);
    }
  };
  int cnt_next = 0, pg_next = 0;
  if (ntile > 0) fetch_meta(t0, cnt_next, pg_next);
  float acc[4];  // dim 32 quad + lane, query rows 4 cgrp .. +3
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = 0.f;
  if (tid < N) corr_s[tid] = 0.f;
  bool alive = true;

  for (int i = 0; i < ntile; ++i) {
    const int st = i % kTcStages;
    const int64_t tile = t0 + i;
    const bool is_group = tile < gt;
    const int64_t r0 = is_group ? tile * TROWS : ws + (tile - gt) * TROWS;  // first row id / position
    const int nvalid = (int)((is_group ? G_vis : ws + wn) - r0 < TROWS ? (is_group ? G_vis : ws + wn) - r0 : TROWS);
    if (tid == 0 && i + kTcStages - 1 < ntile) issue(i + kTcStages - 1);
    // row metadata (log count; -inf = not a row); counts of the next tile prefetched
    const int cnt = cnt_next, pg = pg_next;
    if (i + 1 < ntile) fetch_meta(t0 + i + 1, cnt_next, pg_next);
    float lc = -INFINITY;
    if (tid < nvalid) {
      if (is_group) {
        if (cnt > 0 && cnt <= kChunk) lc = __logf((float)cnt);
        else if (cnt > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
      } else {
        lc = 0.f;
      }
    }
    if (tid < TROWS) {
      lnc_s[tid] = lc;
      cnt_s[tid] = cnt;
      pgs_s[tid] = pg;
    }
    if (!mbar_wait(&full[st], (uint32_t)(i / kTcStages) & 1u, a.status)) alive = false;
    // a row that is not part of the softmax must not feed NaN/Inf into MMA 2
    if (alive && tid < TROWS && lc == -INFINITY) {
      unsigned char* vd = Vring + (size_t)st * kTileBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(vd + h * (kTileBytes / 2) + tid * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      tc::fence_proxy_async();
    }
    tc::fence_before_sync();
    if (!__syncthreads_and(alive)) {
      alive = false;
      break;
    }
    tc::fence_after_sync();
    // ---- MMA 1: S = K_tile . Q^T
    if (tid == 0) {
      const uint32_t kbase = smem_u32(Kring + (size_t)st * kTileBytes);
      const uint32_t id1 = tc::idesc_bf16(TROWS, N, false, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = tc::desc_kmajor_sw128(kbase + (kk / 4) * (kTileBytes / 2) + (kk % 4) * 32);
        const uint64_t bd = tc::desc_kmajor_sw128(smem_u32(Qs) + (kk / 4) * (N * 128) + (kk % 4) * 32);
        tc::mma_bf16(tmem, ad, bd, id1, kk > 0);
      }
      tc::mma_commit(bar_s);
    }
    if (!mbar_wait(bar_s, (uint32_t)i & 1u, a.status)) alive = false;
    tc::fence_after_sync();
    {
      float sv[4];
      tc::tmem_ld4(tmem + ((uint32_t)(32 * quad) << 16) + 4 * cgrp, sv);
#pragma unroll
      for (int c = 0; c < 4; ++c) S_s[(4 * cgrp + c) * TROWS + 32 * quad + lane] = sv[c] * a.scale;
    }
    __syncthreads();
    // ---- query row j (warps j and j + 8, 64 rows each): tile max, weights, sums, top-KG
    if ((warp & 7) < NQ) {
      const int j = warp & 7, half = warp >> 3;
      bool okj = false;
      int64_t tj = 0;
#pragma unroll
      for (int y = 0; y < NQ; ++y)
        if (y == j) {
          okj = ok[y];
          tj = t_row[y];
        }
      float sc[2], lg[2];
      float tmx = -INFINITY;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int row = 64 * half + lane + 32 * q;
        const float lcr = lnc_s[row];
        const bool live = okj && lcr != -INFINITY && (is_group || r0 + row <= tj);
        sc[q] = S_s[j * TROWS + row];
        lg[q] = live ? sc[q] + lcr : -INFINITY;
        tmx = fmaxf(tmx, lg[q]);
      }
      tmx = warp_max(tmx);
      if (lane == 0) pmax_s[half * N + j] = tmx;
      asm volatile("bar.sync %0, 64;" ::"r"(1 + j) : "memory");  // the pair of warps of row j
      tmx = fmaxf(pmax_s[j], pmax_s[N + j]);
      const float mn = fmaxf(m_run, tmx);
      const float corr = m_run == -INFINITY ? 0.f : (mn == -INFINITY ? 1.f : __expf(m_run - mn));
      float psum = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int row = 64 * half + lane + 32 * q;
        const float p = lg[q] == -INFINITY ? 0.f : __expf(lg[q] - mn);
        psum += p;
        *reinterpret_cast<__nv_bfloat16*>(Ps + tc::sw128_offset(j, row, N)) = __float2bfloat16_rn(p);
      }
      psum = warp_sum(psum);
      l_run = l_run * corr + psum;
      m_run = mn;
      if (lane == 0 && half == 0) corr_s[j] = corr;
      if (is_group) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int row = 64 * half + lane + 32 * q;
          float ns = lg[q] != -INFINITY ? sc[q] : -INFINITY;
          int ni = (int)(r0 + row);
          if (ns != -INFINITY && cand_better(ns, ni, ls[KG - 1], lid[KG - 1])) {
            int np = pgs_s[row], nc = cnt_s[row];
#pragma unroll
            for (int k = 0; k < KG; ++k) {
              if (cand_better(ns, ni, ls[k], lid[k])) {
                const float ts = ls[k];
                const int ti = lid[k], tp = lpg[k], tcn = lcn[k];
                ls[k] = ns;
                lid[k] = ni;
                lpg[k] = np;
                lcn[k] = nc;
                ns = ts;
                ni = ti;
                np = tp;
                nc = tcn;
              }
            }
          }
        }
      }
    }
    tc::fence_proxy_async();  // the weights feed MMA 2 through the async proxy
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- MMA 2: O = V_tile^T . P^T  (fresh accumulator)
    if (tid == 0) {
      const uint32_t vbase = smem_u32(Vring + (size_t)st * kTileBytes);
      const uint32_t id2 = tc::idesc_bf16(D, N, true, false);
#pragma unroll
      for (int kk = 0; kk < TROWS / 16; ++kk) {
        const uint64_t ad = tc::desc_mnmajor_sw128(vbase + kk * 2048, kTileBytes / 2);
        const uint64_t bd = tc::desc_kmajor_sw128(smem_u32(Ps) + (kk / 4) * (N * 128) + (kk % 4) * 32);
        tc::mma_bf16(tmem + N, ad, bd, id2, kk > 0);
      }
      tc::mma_commit(bar_o);
    }
    if (!mbar_wait(bar_o, (uint32_t)i & 1u, a.status)) alive = false;
    tc::fence_after_sync();
    {
      float ov[4];
      tc::tmem_ld4(tmem + ((uint32_t)(32 * quad) << 16) + N + 4 * cgrp, ov);
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] = acc[c] * corr_s[4 * cgrp + c] + ov[c];
    }
    tc::fence_before_sync();
    if (!__syncthreads_and(alive)) {
      alive = false;
      break;
    }
  }
  // drain any copy still in flight before the shared memory is released
  if (!alive && tid == 0) {
    for (int i = 0; i < ntile && i < kTcStages; ++i) (void)mbar_wait(&full[i], 0, a.status);
  }

  // ---- outputs: partial states and candidates
  float* part = a.part + ((u * a.nsplit + s) * NQ) * (int64_t)(D + 2);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = 4 * cgrp + c;
    if (j < NQ) part[j * (D + 2) + 2 + 32 * quad + lane] = alive ? acc[c] : 0.f;
  }
  // each query warp merges its lanes' lists (KG rounds of warp argmax over the
  // list heads); the second warp of each pair hands sum and list to the first
  float c_s = -INFINITY;
  int c_i = 0x7fffffff, c_pg = 0, c_cn = 0;
  if ((warp & 7) < NQ) {
    for (int k = 0; k < KG; ++k) {
      float bs = ls[0];
      int bi = lid[0];
      warp_best(bs, bi);
      const unsigned who = __ballot_sync(0xffffffffu, lid[0] == bi && bi != 0x7fffffff);
      const int src = who ? __ffs(who) - 1 : 0;
      const int bp = __shfl_sync(0xffffffffu, lpg[0], src);
      const int bc = __shfl_sync(0xffffffffu, lcn[0], src);
      if (lane == k) {
        c_s = bs;
        c_i = bi;
        c_pg = bp;
        c_cn = bc;
      }
      if (who && lane == src) {  // pop the winner's head
#pragma unroll
        for (int x = 0; x + 1 < KG; ++x) {
          ls[x] = ls[x + 1];
          lid[x] = lid[x + 1];
          lpg[x] = lpg[x + 1];
          lcn[x] = lcn[x + 1];
        }
        ls[KG - 1] = -INFINITY;
        lid[KG - 1] = 0x7fffffff;
      }
    }
  }
  float* xl = S_s;                                         // float [16] sums
  float* xs = S_s + N;                                     // float [16][KG] scores
  int* xi = reinterpret_cast<int*>(S_s + N + N * KG);      // int   [16][KG] ids
  int* xp = xi + N * KG;                                   // int   [16][KG] page ranges
  int* xc = xp + N * KG;                                   // int   [16][KG] counts
  __syncthreads();
  if (warp >= 8 && (warp & 7) < NQ) {
    const int j = warp & 7;
    if (lane == 0) xl[j] = l_run;
    if (lane < KG) {
      xs[j * KG + lane] = c_s;
      xi[j * KG + lane] = c_i;
      xp[j * KG + lane] = c_pg;
      xc[j * KG + lane] = c_cn;
    }
  }
  __syncthreads();
  if (warp < NQ) {
    const int j = warp;
    // the two sorted lists sit in lanes 0..KG-1 (this warp) and KG..2KG-1 (partner)
    float hs = c_s;
    int hi = c_i, hp = c_pg, hc = c_cn;
    if (lane >= KG && lane < 2 * KG) {
      hs = xs[j * KG + lane - KG];
      hi = xi[j * KG + lane - KG];
      hp = xp[j * KG + lane - KG];
      hc = xc[j * KG + lane - KG];
    } else if (lane >= 2 * KG) {
      hs = -INFINITY;
      hi = 0x7fffffff;
    }
    float os = -INFINITY;
    int oi = 0x7fffffff, op = 0, oc = 0;
    for (int k = 0; k < KG; ++k) {
      float bs = hs;
      int bi = hi;
      warp_best(bs, bi);
      const unsigned who = __ballot_sync(0xffffffffu, hi == bi && bi != 0x7fffffff);
      const int src = who ? __ffs(who) - 1 : 0;
      const int bp = __shfl_sync(0xffffffffu, hp, src);
      const int bc = __shfl_sync(0xffffffffu, hc, src);
      if (lane == k) {
        os = bs;
        oi = bi;
        op = bp;
        oc = bc;
      }
      if (who && lane == src) {
        hs = -INFINITY;
        hi = 0x7fffffff;
      }
    }
    if (lane == 0) {
      part[j * (D + 2) + 0] = alive ? m_run : -INFINITY;
      part[j * (D + 2) + 1] = alive ? l_run + xl[j] : 0.f;
    }
    Cand* out = reinterpret_cast<Cand*>(a.cand) + ((u * a.nsplit + s) * NQ + j) * KG;
    if (lane < KG) {
      Cand c;
      const bool none = !alive || oi == 0x7fffffff;
      c.s = none ? -INFINITY : os;
      c.id = none ? -1 : oi;
      c.pages = none ? 0 : op;
      c.cnt = none ? 0 : oc;
      out[lane] = c;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 32);
  pdl_launch_dependents();
}

template <int NQ>
cudaError_t launch_nq(const AttendArgs& a, const TcMaps& maps, cudaStream_t stream) {
  auto kern = a.G <= 8 ? scan_tc_kernel<NQ, 8> : scan_tc_kernel<NQ, 16>;
  const size_t smem = TcSmem::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)a.units, (unsigned)a.nsplit), kTcThreads, smem, stream>>>(maps, a);
  return cudaGetLastError();
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
