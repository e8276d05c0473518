// lod_attend.cu -- LoD decode and prefill attention ("Level of Detail
// Attention", How It Works, paragraphs 2-3).
//
// Two kernels per batch of query rows:
//
//  scan    grid (unit, split).  A unit is one KV head of one sequence with its
//          NQ query rows (decode: the g query heads; prefill: g heads x NP
//          positions).  A split stages a slice of rows in shared memory with
//          TMA bulk copies -- either visible group summaries (mean key, mean
//          value, count) or exact window/sink tokens -- and computes
//            pass 1  the scores of all its rows against the NQ queries,
//            then    per query row the max logit (score + ln count) and, for
//                    group slices, the local top-KG groups by score,
//            pass 2  the weighted sum of its values,
//          leaving a partial softmax state (max, sum, acc[d]) over ALL its rows.
//  refine  one CTA per query row, launched as a programmatic dependent of the
//          scan.  It merges the split states, picks the global top
//          `top_groups` groups from the local candidates, removes those groups'
//          coarse terms (they are replaced by finer entries), scores each
//          opened group's page summaries, opens the top `top_pages` pages and
//          adds their tokens exactly (values staged by TMA), adds the other
//          pages as coarse entries (page mean logit + ln count, page mean
//          value), and writes out = acc / sum and the log-sum-exp.
//
// Removing the opened groups after the fact (instead of holding them out of
// the scan) is numerically safe: the entries that replace an opened group --
// its pages, or their tokens -- carry at least the group's own mass (the
// method's "conservative estimate" property: n exp(q.mean k) <= sum exp(q.k)),
// so the final normaliser is never smaller than what was subtracted and the
// cancellation error stays at the fp32 rounding level of the output.
#include "lod_internal.cuh"

namespace lod {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& raw, float* f) {
  if constexpr (sizeof(T) == 4) {
    f[0] = __uint_as_float(raw.x);
    f[1] = __uint_as_float(raw.y);
    f[2] = __uint_as_float(raw.z);
    f[3] = __uint_as_float(raw.w);
  } else {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// Dot product of a whole d-row (owned by one lane) with q held in shared memory.
template <typename T, int D>
__device__ __forceinline__ float row_dot(const T* __restrict__ row, const float* __restrict__ qs) {
  constexpr int VEC = 16 / sizeof(T);
  uint4 raw[D / VEC];
#pragma unroll
  for (int v = 0; v < D / VEC; ++v) raw[v] = __ldg(reinterpret_cast<const uint4*>(row) + v);
  float2 s = make_float2(0.f, 0.f);
#pragma unroll
  for (int v = 0; v < D / VEC; ++v) {
    float f[VEC];
    unpack16<T>(raw[v], f);
#pragma unroll
    for (int e = 0; e < VEC; e += 2)
      s = ffma2(make_float2(qs[v * VEC + e], qs[v * VEC + e + 1]), make_float2(f[e], f[e + 1]), s);
  }
  return s.x + s.y;
}

struct UnitInfo {
  int b, kvh;
  int64_t blk, nblk;
};

__device__ __forceinline__ UnitInfo unit_info(const AttendArgs& a, int64_t u) {
  UnitInfo ui;
  if (a.seq_lens) {
    ui.b = (int)(u / a.Hkv);
    ui.kvh = (int)(u % a.Hkv);
    ui.blk = 0;
    ui.nblk = 1;
  } else {
    ui.nblk = (a.pos_hi - a.pos_lo + a.NP - 1) / a.NP;
    ui.b = (int)(u / (a.Hkv * ui.nblk));
    ui.kvh = (int)((u / ui.nblk) % a.Hkv);
    ui.blk = u % ui.nblk;
  }
  return ui;
}

// Candidate record written by the scan and read by the refine kernel.
struct Cand {
  float s;     // scale * q.mean_k
  int id;      // global group id (chunk * k + slot), -1 = none
  int pages;   // first page slot | (last page slot + 1) << 16
  int cnt;     // group size
};

// ------------------------------------------------------------------ scan

template <typename T, int D, int NQ>
struct ScanSmem {
  static constexpr int R = kScanRows;
  static constexpr size_t kv_bytes = (size_t)R * D * sizeof(T);
  static constexpr size_t off_V = kv_bytes;
  static constexpr size_t off_S = 2 * kv_bytes;                        // float [NQ][R]
  static constexpr size_t off_P = off_S + sizeof(float) * NQ * R;      // float [R][NQ]
  static constexpr size_t off_lnc = off_P + sizeof(float) * NQ * R;    // float [R]
  static constexpr size_t off_pos = off_lnc + sizeof(float) * R;       // int64 [R]
  static constexpr size_t off_m = off_pos + sizeof(int64_t) * R;       // float [NQ]
  static constexpr size_t off_l = off_m + sizeof(float) * 16;          // float [NQ]
  static constexpr size_t off_bar = off_l + sizeof(float) * 16;        // uint64 [2]
  static constexpr size_t bytes = off_bar + 16;
  static_assert(sizeof(float) * kWarps * NQ * D <= kv_bytes, "reduction scratch reuses the K stage");
};

template <typename T, int D, int NQ, int KG>
__global__ void __launch_bounds__(kThreads, 2) scan_kernel(AttendArgs a) {
  constexpr int EPL = 16 / sizeof(T);  // elements per lane per 16-byte load
  constexpr int LPR = D / EPL;         // lanes per row
  constexpr int RPI = 32 / LPR;        // rows per warp per step
  constexpr int R = kScanRows;
  constexpr int ROWB = D * sizeof(T);
  using SM = ScanSmem<T, D, NQ>;
  static_assert(NQ <= LPR, "each query row's score must land on its own lanes");

  const int64_t u = blockIdx.x;
  const int s = blockIdx.y;
  const int nsplit = a.nsg + a.nsw;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int li = lane % LPR, sub = lane / LPR;
  const UnitInfo ui = unit_info(a, u);

  extern __shared__ __align__(128) unsigned char smem[];
  T* Ks = reinterpret_cast<T*>(smem);
  T* Vs = reinterpret_cast<T*>(smem + SM::off_V);
  float* S_s = reinterpret_cast<float*>(smem + SM::off_S);
  float* P_s = reinterpret_cast<float*>(smem + SM::off_P);
  float* lnc_s = reinterpret_cast<float*>(smem + SM::off_lnc);
  int64_t* pos_s = reinterpret_cast<int64_t*>(smem + SM::off_pos);
  float* m_s = reinterpret_cast<float*>(smem + SM::off_m);
  float* l_s = reinterpret_cast<float*>(smem + SM::off_l);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM::off_bar);
  float* red = reinterpret_cast<float*>(smem);  // [kWarps][NQ][D], after pass 1

  // ---- the unit's query rows: positions and validity
  int64_t t_row[NQ];
  bool ok[NQ];
  int64_t t_max = -1;
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    if (a.seq_lens) {
      const int64_t L = a.seq_lens[ui.b];
      ok[r] = (r < a.g) && L >= 1 && L <= a.Tmax;
      t_row[r] = L - 1;
    } else {
      const int64_t pi = a.pos_lo + ui.blk * a.NP + r / a.g;
      ok[r] = (r < a.g * a.NP) && pi < a.pos_hi;
      t_row[r] = a.q_begin + pi;
    }
    if (ok[r] && t_row[r] > t_max) t_max = t_row[r];
  }
  if (a.seq_lens && t_max < 0 && s == 0 && tid == 0) set_status(a.status, LOD_ST_BAD_SEQLEN);

  // ---- rows of this split
  const int64_t unit_kv = (int64_t)ui.b * a.Hkv + ui.kvh;
  const bool is_group = s < a.nsg;
  int64_t lo = 0, ws = 0;
  int nrows = 0, ns = 0;
  int64_t wb = 0;
  if (t_max >= 0) {
    const int64_t bt = t_max / kChunk;
    const int64_t nw = a.window / kChunk;
    wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;  // visible chunks [0, wb)
    ws = wb * kChunk;                        // window start
    if (is_group) {
      const int64_t G_vis = wb * a.k;
      const int64_t per = (G_vis + a.nsg - 1) / a.nsg;
      lo = s * per;
      const int64_t hi = lo + per < G_vis ? lo + per : G_vis;
      nrows = hi > lo ? (int)(hi - lo) : 0;
    } else {
      // window list: the sinks, then [ws, t_max]
      const int64_t nsk = a.sinks < ws ? a.sinks : ws;
      const int64_t total = nsk + (t_max - ws + 1);
      const int64_t per = (total + a.nsw - 1) / a.nsw;
      const int64_t e0 = (int64_t)(s - a.nsg) * per;
      const int64_t e1 = e0 + per < total ? e0 + per : total;
      nrows = e1 > e0 ? (int)(e1 - e0) : 0;
      lo = e0;       // first list index
      ns = (int)nsk; // list indices < ns are sinks
    }
  }
  const T* Kb = static_cast<const T*>(a.K) + ui.b * a.sb + ui.kvh * a.sh;
  const T* Vb = static_cast<const T*>(a.V) + ui.b * a.sb + ui.kvh * a.sh;
  const T* gK = static_cast<const T*>(a.gK) + unit_kv * a.Cmax * a.k * D;
  const T* gV = static_cast<const T*>(a.gV) + unit_kv * a.Cmax * a.k * D;
  const int32_t* gC = a.gCnt + unit_kv * a.Cmax * a.k;

  // ---- stage the rows in shared memory: two pipeline stages of TMA bulk copies
  const int n0 = nrows < R / 2 ? nrows : R / 2;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0 && nrows > 0) {
    for (int st = 0; st < 2; ++st) {
      const int r0 = st ? n0 : 0, r1 = st ? nrows : n0;
      if (r1 <= r0) continue;
      if (lane == 0) mbar_arrive_expect(&bar[st], (uint32_t)(r1 - r0) * 2u * ROWB);
      __syncwarp();
      if (is_group) {
        if (lane == 0) {
          bulk_g2s(Ks + r0 * D, gK + (lo + r0) * D, (uint32_t)(r1 - r0) * ROWB, &bar[st]);
          bulk_g2s(Vs + r0 * D, gV + (lo + r0) * D, (uint32_t)(r1 - r0) * ROWB, &bar[st]);
        }
      } else {
        for (int r = r0 + lane; r < r1; r += 32) {
          const int64_t e = lo + r;
          const int64_t pos = e < ns ? e : ws + (e - ns);
          bulk_g2s(Ks + r * D, Kb + pos * a.st, ROWB, &bar[st]);
          bulk_g2s(Vs + r * D, Vb + pos * a.st, ROWB, &bar[st]);
        }
      }
    }
  }
  // per-row log-count (group rows) and position (window rows), -inf = skip
  for (int r = tid; r < R; r += kThreads) {
    float lc = -INFINITY;
    int64_t pos = -1;
    if (r < nrows) {
      if (is_group) {
        const int cnt = gC[lo + r];
        if (cnt > 0 && cnt <= kChunk) lc = __logf((float)cnt);
        else if (cnt > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
      } else {
        const int64_t e = lo + r;
        pos = e < ns ? e : ws + (e - ns);
        lc = 0.f;
      }
    }
    lnc_s[r] = lc;
    pos_s[r] = pos;
  }

  // ---- the query rows (pre-scaled): this lane's EPL dims of each
  float2 q2[NQ][EPL / 2];
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    float f[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) f[e] = 0.f;
    if (ok[r]) {
      const int hq = ui.kvh * a.g + (r % a.g);
      const int64_t pi = a.seq_lens ? 0 : a.pos_lo + ui.blk * a.NP + r / a.g;
      const T* qp = static_cast<const T*>(a.q) + (((int64_t)ui.b * a.Hq + hq) * a.Tq + pi) * D;
      load_f<T, EPL>(qp + li * EPL, f);
    }
#pragma unroll
    for (int e = 0; e < EPL; e += 2) q2[r][e / 2] = make_float2(f[e] * a.scale, f[e + 1] * a.scale);
  }
  __syncthreads();

  // ---- pass 1: scores.  Lanes of a row own EPL dims each; a reduce-scatter
  // over the row's LPR lanes leaves query row h's score on lanes
  // h * (LPR/NQ) .. (h+1) * (LPR/NQ) - 1.
  bool ok_stage[2] = {true, true};
  for (int base = 0; base < nrows; base += kWarps * RPI) {
    const int row = base + warp * RPI + sub;
    const int st = base >= n0 ? 1 : 0;
    if (!ok_stage[st]) break;
    if (!mbar_wait(&bar[st], 0, a.status)) {
      ok_stage[st] = false;
      break;
    }
    const bool valid = row < nrows;
    float k[EPL];
    if (valid) {
      uint4 raw = *reinterpret_cast<const uint4*>(Ks + row * D + li * EPL);
      unpack16<T>(raw, k);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) k[e] = 0.f;
    }
    float part[NQ];
#pragma unroll
    for (int r = 0; r < NQ; ++r) {
      float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < EPL; e += 2) acc2 = ffma2(q2[r][e / 2], make_float2(k[e], k[e + 1]), acc2);
      part[r] = acc2.x + acc2.y;
    }
#pragma unroll
    for (int step = 0; step < ilog2(LPR); ++step) {
      const int m = LPR >> (step + 1);
      constexpr int dummy = 0;
      (void)dummy;
      const int n = NQ >> step;  // live values before this step
      if (n > 1) {
        const bool upper = (li & m) != 0;
#pragma unroll
        for (int i = 0; i < NQ / 2; ++i) {
          if (i < n / 2) {
            const float send = upper ? part[i] : part[i + n / 2];
            const float keep = upper ? part[i + n / 2] : part[i];
            part[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
        }
      } else {
        part[0] += __shfl_xor_sync(0xffffffffu, part[0], m);
      }
    }
    constexpr int SHIFT = ilog2(LPR) - ilog2(NQ);
    if (valid && (li & ((1 << SHIFT) - 1)) == 0) S_s[(li >> SHIFT) * R + row] = part[0];
  }
  // every thread must see both stages complete before pass 2 and before exit
  for (int st = 0; st < 2; ++st) {
    const bool used = st ? nrows > n0 : nrows > 0;
    if (used && ok_stage[st] && !mbar_wait(&bar[st], 0, a.status)) ok_stage[st] = false;
  }
  const bool staged = ok_stage[0] && ok_stage[1];
  __syncthreads();

  // ---- per query row: max logit, and (group slices) the local top-KG
  if (warp < NQ) {
    const int r = warp;
    float mx = -INFINITY;
    for (int e = lane; e < nrows; e += 32) {
      const bool live = ok[r] && staged && lnc_s[e] != -INFINITY && (is_group || pos_s[e] <= t_row[r]);
      if (live) mx = fmaxf(mx, S_s[r * R + e] + lnc_s[e]);
    }
    mx = warp_max(mx);
    if (lane == 0) m_s[r] = mx;
    if (is_group) {
      constexpr int PER = R / 32;
      float cs[PER];
      int cid[PER];
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = lane + 32 * j;
        const bool live = ok[r] && staged && e < nrows && lnc_s[e] != -INFINITY;
        cs[j] = live ? S_s[r * R + e] : -INFINITY;
        cid[j] = live ? (int)(lo + e) : 0x7fffffff;
      }
      Cand* out = reinterpret_cast<Cand*>(a.cand) + ((u * a.nsg + s) * NQ + r) * KG;
      for (int rank = 0; rank < KG; ++rank) {
        float bs = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < PER; ++j)
          if (cand_better(cs[j], cid[j], bs, bi)) {
            bs = cs[j];
            bi = cid[j];
          }
        warp_best(bs, bi);
#pragma unroll
        for (int j = 0; j < PER; ++j)
          if (cid[j] == bi) {
            cs[j] = -INFINITY;
            cid[j] = 0x7fffffff;
          }
        if (lane == rank) {
          Cand c;
          if (bi == 0x7fffffff) {
            c.s = -INFINITY;
            c.id = -1;
            c.pages = 0;
            c.cnt = 0;
          } else {
            const int64_t ch = bi / a.k;
            const int j = bi % a.k;
            const int16_t* gp = a.gPage + unit_kv * a.Cmax * (a.k + 1) + ch * (a.k + 1) + j;
            c.s = bs;
            c.id = bi;
            c.pages = ((int)(uint16_t)gp[0]) | ((int)(uint16_t)gp[1] << 16);
            c.cnt = gC[bi];
          }
          out[rank] = c;
        }
      }
    }
  }
  __syncthreads();

  // ---- softmax weights of every (row, query row) pair
  for (int idx = tid; idx < R * NQ; idx += kThreads) {
    const int e = idx / NQ, r = idx % NQ;
    float p = 0.f;
    if (e < nrows && ok[r] && staged && lnc_s[e] != -INFINITY && (is_group || pos_s[e] <= t_row[r]))
      p = __expf(S_s[r * R + e] + lnc_s[e] - m_s[r]);
    P_s[e * NQ + r] = p;
  }
  __syncthreads();
  if (warp < NQ) {
    float sum = 0.f;
    for (int e = lane; e < nrows; e += 32) sum += P_s[e * NQ + warp];
    sum = warp_sum(sum);
    if (lane == 0) l_s[warp] = sum;
  }

  // ---- pass 2: acc[r][:] += P[row][r] * V[row][:]
  float2 acc[NQ][EPL / 2];
#pragma unroll
  for (int r = 0; r < NQ; ++r)
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) acc[r][e] = make_float2(0.f, 0.f);
  if (staged) {
    for (int base = 0; base < nrows; base += kWarps * RPI) {
      const int row = base + warp * RPI + sub;
      if (row < nrows && lnc_s[row] != -INFINITY) {
        float v[EPL];
        uint4 raw = *reinterpret_cast<const uint4*>(Vs + row * D + li * EPL);
        unpack16<T>(raw, v);
        float p[NQ];
#pragma unroll
        for (int r = 0; r < NQ; r += 4) {
          if constexpr (NQ % 4 == 0) {
            const float4 pp = *reinterpret_cast<const float4*>(P_s + row * NQ + r);
            p[r] = pp.x;
            p[r + 1] = pp.y;
            p[r + 2] = pp.z;
            p[r + 3] = pp.w;
          } else {
#pragma unroll
            for (int x = 0; x < 4 && r + x < NQ; ++x) p[r + x] = P_s[row * NQ + r + x];
          }
        }
#pragma unroll
        for (int r = 0; r < NQ; ++r)
#pragma unroll
          for (int e = 0; e < EPL; e += 2)
            acc[r][e / 2] = ffma2(make_float2(p[r], p[r]), make_float2(v[e], v[e + 1]), acc[r][e / 2]);
      }
    }
  }
  // the warp's rows-per-step slices hold separate sums: fold them
#pragma unroll
  for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
    for (int r = 0; r < NQ; ++r)
#pragma unroll
      for (int e = 0; e < EPL / 2; ++e) {
        acc[r][e].x += __shfl_xor_sync(0xffffffffu, acc[r][e].x, m);
        acc[r][e].y += __shfl_xor_sync(0xffffffffu, acc[r][e].y, m);
      }
  __syncthreads();  // the K stage becomes the cross-warp reduction buffer
  if (sub == 0) {
#pragma unroll
    for (int r = 0; r < NQ; ++r)
#pragma unroll
      for (int e = 0; e < EPL; e += 4)
        *reinterpret_cast<float4*>(red + (warp * NQ + r) * D + li * EPL + e) =
            make_float4(acc[r][e / 2].x, acc[r][e / 2].y, acc[r][e / 2 + 1].x, acc[r][e / 2 + 1].y);
  }
  __syncthreads();
  float* part = a.part + ((u * nsplit + s) * NQ) * (int64_t)(D + 2);
  for (int idx = tid; idx < NQ * (D + 2); idx += kThreads) {
    const int r = idx / (D + 2), c = idx % (D + 2);
    float v;
    if (c == 0) {
      v = m_s[r];
    } else if (c == 1) {
      v = l_s[r];
    } else {
      v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[(w * NQ + r) * D + (c - 2)];
    }
    part[idx] = v;
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ refine

template <typename T, int D>
struct RefineSmem {
  static constexpr int ROWB = D * sizeof(T);
  static constexpr int kRows = 48;  // per warp: 32 exact tokens + 16 coarse page means
  static constexpr size_t off_V = 0;                                     // [kWarps][kRows][D] T
  static constexpr size_t off_perm = (size_t)kWarps * kRows * ROWB;      // int16 [kWarps][kChunk]
  static constexpr size_t off_q = off_perm + 2 * kWarps * kChunk;        // float [D]
  static constexpr size_t off_g = off_q + sizeof(float) * D;            // float [D+2]
  static constexpr size_t off_w = off_g + sizeof(float) * (D + 4);      // float [kWarps][D+2]
  static constexpr size_t off_d = off_w + sizeof(float) * kWarps * (D + 4);  // float [kWarps][D+2]
  static constexpr size_t off_c = off_d + sizeof(float) * kWarps * (D + 4);  // Cand [kMaxTopGroups]
  static constexpr size_t off_bar = off_c + sizeof(Cand) * kMaxTopGroups + 16;
  static constexpr size_t bytes = off_bar + 8 * kWarps + 16;
};

template <typename T, int D, int NQ, int KG>
__global__ void __launch_bounds__(kThreads, 2) refine_kernel(AttendArgs a) {
  constexpr int DPL = D / 32;
  constexpr int ROWB = D * sizeof(T);
  using SM = RefineSmem<T, D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nsplit = a.nsg + a.nsw;
  const int64_t npos = a.seq_lens ? 1 : a.pos_hi - a.pos_lo;
  const int64_t row = blockIdx.x;
  const int b = (int)(row / (a.Hq * npos));
  const int hq = (int)((row / npos) % a.Hq);
  const int64_t pi = a.seq_lens ? 0 : a.pos_lo + row % npos;
  const int kvh = hq / a.g, hh = hq % a.g;
  int64_t u;
  int r;
  if (a.seq_lens) {
    u = (int64_t)b * a.Hkv + kvh;
    r = hh;
  } else {
    const int64_t nblk = (a.pos_hi - a.pos_lo + a.NP - 1) / a.NP;
    const int64_t rel = pi - a.pos_lo;
    u = ((int64_t)b * a.Hkv + kvh) * nblk + rel / a.NP;
    r = (int)(rel % a.NP) * a.g + hh;
  }
  const int64_t orow = ((int64_t)b * a.Hq + hq) * a.Tq + pi;  // row of q / out / lse
  T* out = static_cast<T*>(a.out) + orow * D;
  const int64_t unit_kv = (int64_t)b * a.Hkv + kvh;

  extern __shared__ __align__(128) unsigned char smem[];
  T* Vst = reinterpret_cast<T*>(smem + SM::off_V);
  int16_t* perm_s = reinterpret_cast<int16_t*>(smem + SM::off_perm);
  float* qs = reinterpret_cast<float*>(smem + SM::off_q);
  float* gstate = reinterpret_cast<float*>(smem + SM::off_g);
  float* wstate = reinterpret_cast<float*>(smem + SM::off_w);
  float* dstate = reinterpret_cast<float*>(smem + SM::off_d);
  Cand* win = reinterpret_cast<Cand*>(smem + SM::off_c);
  int* nwin_s = reinterpret_cast<int*>(smem + SM::off_c + sizeof(Cand) * kMaxTopGroups);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM::off_bar);

  // ---- prologue (overlaps the scan's tail): position, q, barriers
  const int64_t t = a.seq_lens ? a.seq_lens[b] - 1 : a.q_begin + pi;
  if (t < 0 || t >= a.Tmax) {  // invalid sequence length (decode)
    for (int i = tid; i < D; i += kThreads) out[i] = Elem<T>::from_f(0.f);
    if (tid == 0) {
      set_status(a.status, LOD_ST_BAD_SEQLEN);
      if (a.lse) a.lse[orow] = -INFINITY;
    }
    if (a.sel_groups)
      for (int i = tid; i < a.G; i += kThreads) a.sel_groups[orow * a.G + i] = -1;
    if (a.sel_pages)
      for (int i = tid; i < a.G * a.TP; i += kThreads) a.sel_pages[orow * a.G * a.TP + i] = -1;
    return;
  }
  {
    const T* qp = static_cast<const T*>(a.q) + orow * D;
    for (int i = tid; i < D; i += kThreads) qs[i] = Elem<T>::to_f(qp[i]) * a.scale;
  }
  if (tid < kWarps) mbar_init(&bar[tid], 1);
  if (tid == 0) fence_mbar_init();
  pdl_wait();  // the scan's partial states and candidates are visible from here on

  // ---- global top-G over the group splits' candidates (warp 0)
  if (warp == 0) {
    const int ncand = a.nsg * KG;
    const Cand* src = reinterpret_cast<const Cand*>(a.cand) + (u * a.nsg * NQ) * (int64_t)KG;
    float lastS = INFINITY;
    int lastI = -1;
    int nwin = 0;
    for (int rank = 0; rank < a.G; ++rank) {
      float bs = -INFINITY;
      int bi = 0x7fffffff, bidx = -1;
      for (int e = lane; e < ncand; e += 32) {
        const int sp = e / KG, j = e % KG;
        const Cand* c = src + ((int64_t)sp * NQ + r) * KG + j;
        const int id = c->id;
        if (id < 0) continue;
        const float sc = c->s;
        const bool after = rank == 0 || cand_better(lastS, lastI, sc, id);
        if (after && cand_better(sc, id, bs, bi)) {
          bs = sc;
          bi = id;
          bidx = (int)(((int64_t)sp * NQ + r) * KG + j);
        }
      }
      float ws_ = bs;
      int wi_ = bi;
      warp_best(ws_, wi_);
      if (wi_ == 0x7fffffff) break;
      if (bi == wi_) win[rank] = src[bidx];
      lastS = ws_;
      lastI = wi_;
      ++nwin;
    }
    if (lane == 0) *nwin_s = nwin;
  } else {
    // ---- merge the split states (thread c owns component c: m, l, acc[])
    const float* ps = a.part + (u * nsplit * NQ + r) * (int64_t)(D + 2);
    const int64_t stride = (int64_t)NQ * (D + 2);
    float M = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, ps[sp * stride]);
    for (int c = tid - 32; c < D + 2; c += kThreads - 32) {
      float v = 0.f;
      if (c == 0) {
        v = M;
      } else {
        for (int sp = 0; sp < nsplit; ++sp) {
          const float ms = ps[sp * stride];
          if (ms != -INFINITY) v = fmaf(ps[sp * stride + c], __expf(ms - M), v);
        }
      }
      gstate[c] = v;
    }
  }
  __syncthreads();
  const int nwin = *nwin_s;
  const float M = gstate[0];

  // ---- per opened group (warp w: groups w, w + 8, ...)
  float m = -INFINITY, l = 0.f, acc[DPL];
  float dl = 0.f, dacc[DPL];  // the opened groups' coarse terms, to remove (relative to M)
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = dacc[i] = 0.f;
  const T* gV = static_cast<const T*>(a.gV) + unit_kv * a.Cmax * a.k * D;
  const T* pK = static_cast<const T*>(a.pK) + unit_kv * a.Cmax * a.P * D;
  const T* pV = static_cast<const T*>(a.pV) + unit_kv * a.Cmax * a.P * D;
  const int32_t* pC = a.pCnt + unit_kv * a.Cmax * a.P;
  const int16_t* pB = a.pBeg + unit_kv * a.Cmax * a.P;
  const int16_t* pm = a.perm + unit_kv * a.Cmax * kChunk;
  const T* Kb = static_cast<const T*>(a.K) + b * a.sb + kvh * a.sh;
  const T* Vb = static_cast<const T*>(a.V) + b * a.sb + kvh * a.sh;
  T* myV = Vst + warp * SM::kRows * D;
  int16_t* myperm = perm_s + warp * kChunk;
  uint32_t phase = 0;
  for (int w = warp; w < nwin; w += kWarps) {
    const Cand cw = win[w];
    const int64_t c = cw.id / a.k;
    const int p0 = cw.pages & 0xffff, p1 = (cw.pages >> 16) & 0xffff;
    int open_slot[kMaxTopPages];
#pragma unroll
    for (int x = 0; x < kMaxTopPages; ++x) open_slot[x] = -1;
    // remove this group's coarse term: exp(s + ln n - M) * (1, gV)
    if (cw.cnt > 0 && cw.cnt <= kChunk) {
      const float e = __expf(cw.s + __logf((float)cw.cnt) - M);
      float gv[DPL];
      load_f<T, DPL>(gV + (int64_t)cw.id * D + lane * DPL, gv);
      dl -= e;
#pragma unroll
      for (int i = 0; i < DPL; ++i) dacc[i] = fmaf(-e, gv[i], dacc[i]);
    } else {
      if (lane == 0) set_status(a.status, LOD_ST_BAD_COUNT);
    }
    if (p1 < p0 || p1 > a.P || p1 - p0 > 32) {
      if (lane == 0) set_status(a.status, LOD_ST_BAD_PAGE);
    } else {
      const int np = p1 - p0;
      // the chunk's member list, and lane p's page summary score
      *reinterpret_cast<uint4*>(myperm + lane * 8) =
          __ldg(reinterpret_cast<const uint4*>(pm + c * kChunk) + lane);
      float sc = -INFINITY;
      int cntp = 0, begp = 0;
      if (lane < np) {
        cntp = pC[c * a.P + p0 + lane];
        begp = pB[c * a.P + p0 + lane];
        sc = row_dot<T, D>(pK + (c * a.P + p0 + lane) * D, qs);
      }
      __syncwarp();
      // top-TP pages by (score desc, slot asc)
      float s2 = sc;
      int sl2 = lane < np ? p0 + lane : 0x7fffffff;
      int nopen = 0;
      for (int x = 0; x < a.TP && x < np; ++x) {
        float bs = s2;  // (the chunk-member list is in shared memory after the __syncwarp above)
        int bi = sl2;
        warp_best(bs, bi);
        open_slot[x] = bi;
        if (sl2 == bi) {
          s2 = -INFINITY;
          sl2 = 0x7fffffff;
        }
        ++nopen;
      }
      bool is_open = false;
#pragma unroll
      for (int x = 0; x < kMaxTopPages; ++x) is_open |= (open_slot[x] == p0 + lane);
      // coarse entries: the unopened pages of this group (lane p), staged with the first batch
      const bool cv = lane < np && !is_open && cntp > 0 && cntp <= kPage;
      if (lane < np && !is_open && (cntp <= 0 || cntp > kPage)) set_status(a.status, LOD_ST_BAD_COUNT);
      const unsigned cm = __ballot_sync(0xffffffffu, cv);
      const float lgc = cv ? sc + __logf((float)cntp) : -INFINITY;
      // exact members of the opened pages, 32 per batch: lane e -> (page e/16, member e%16)
      const int nbatch = (nopen * kPage + 31) / 32;
      for (int bt = 0; bt < (nbatch > 0 ? nbatch : 1); ++bt) {
        const int e = bt * 32 + lane;
        const int x = e / kPage, mi = e % kPage;
        int slot = -1;
#pragma unroll
        for (int y = 0; y < kMaxTopPages; ++y)
          if (y == x) slot = open_slot[y];
        const int sl_lane = slot >= 0 ? slot - p0 : 0;
        const int n_of = __shfl_sync(0xffffffffu, cntp, sl_lane & 31);
        const int b_of = __shfl_sync(0xffffffffu, begp, sl_lane & 31);
        bool ev = x < nopen && slot >= 0 && mi < n_of;
        if (ev && (n_of > kPage || b_of < 0 || b_of + n_of > kChunk)) {
          set_status(a.status, LOD_ST_BAD_PAGE);
          ev = false;
        }
        const int off = ev ? myperm[b_of + mi] : 0;
        if (ev && (off < 0 || off >= kChunk)) {
          set_status(a.status, LOD_ST_BAD_MEMBER);
          ev = false;
        }
        const int64_t pos = c * kChunk + off;
        const bool cvb = bt == 0 && cv;
        const unsigned vm = __ballot_sync(0xffffffffu, ev);
        const unsigned cmb = bt == 0 ? cm : 0u;
        // value rows (exact tokens and coarse page means) go to shared memory by
        // TMA while the key rows are dotted in registers
        if (lane == 0 && (vm | cmb)) mbar_arrive_expect(&bar[warp], (uint32_t)(__popc(vm) + __popc(cmb)) * ROWB);
        __syncwarp();
        if (ev) bulk_g2s(myV + lane * D, Vb + pos * a.st, ROWB, &bar[warp]);
        if (cvb) bulk_g2s(myV + (32 + lane) * D, pV + (c * a.P + p0 + lane) * D, ROWB, &bar[warp]);
        const float lge = ev ? row_dot<T, D>(Kb + pos * a.st, qs) : -INFINITY;
        const float lgcb = cvb ? lgc : -INFINITY;
        const float bm = warp_max(fmaxf(lge, lgcb));
        if (bm == -INFINITY) continue;  // nothing staged in this batch
        const float mn = fmaxf(m, bm);
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        const float pe = ev ? __expf(lge - mn) : 0.f;
        const float pc = cvb ? __expf(lgcb - mn) : 0.f;
        l = l * corr + warp_sum(pe + pc);
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] *= corr;
        m = mn;
        const bool okw = mbar_wait(&bar[warp], phase, a.status);
        phase ^= 1u;
        if (!okw) {
          (void)mbar_wait(&bar[warp], phase ^ 1u, a.status);  // drain before the buffer is reused
          __syncwarp();
          continue;
        }
        for (int j = 0; j < 64; ++j) {
          const bool on = j < 32 ? ((vm >> j) & 1u) : ((cmb >> (j - 32)) & 1u);
          if (!on) continue;
          const float pj = __shfl_sync(0xffffffffu, j < 32 ? pe : pc, j & 31);
          float v[DPL];
          if constexpr (sizeof(T) == 2 && DPL == 4) {
            const uint2 rw = *reinterpret_cast<const uint2*>(myV + j * D + lane * DPL);
            v[0] = __uint_as_float(rw.x << 16);
            v[1] = __uint_as_float(rw.x & 0xffff0000u);
            v[2] = __uint_as_float(rw.y << 16);
            v[3] = __uint_as_float(rw.y & 0xffff0000u);
          } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) v[i] = Elem<T>::to_f(myV[j * D + lane * DPL + i]);
          }
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, v[i], acc[i]);
        }
        __syncwarp();
      }
    }
    if (a.sel_pages && lane < a.TP) {
      int32_t v = -1;
#pragma unroll
      for (int x = 0; x < kMaxTopPages; ++x)
        if (x == lane && open_slot[x] >= 0) v = (int32_t)(c * a.P + open_slot[x]);
      a.sel_pages[(orow * a.G + w) * a.TP + lane] = v;
    }
  }

  // ---- final merge: scan state (max M) + per-warp fine states + removals
  float* ws_ = wstate + warp * (D + 4);
  float* ds_ = dstate + warp * (D + 4);
  if (lane == 0) {
    ws_[0] = m;
    ws_[1] = l;
    ds_[0] = dl;
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    ws_[2 + lane * DPL + i] = acc[i];
    ds_[2 + lane * DPL + i] = dacc[i];
  }
  __syncthreads();
  float MM = M;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) MM = fmaxf(MM, wstate[w * (D + 4)]);
  const float cM = __expf(M - MM);
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float mw = wstate[w * (D + 4)];
    if (mw != -INFINITY) L = fmaf(wstate[w * (D + 4) + 1], __expf(mw - MM), L);
    L = fmaf(dstate[w * (D + 4)], cM, L);
  }
  L = fmaf(gstate[1], cM, L);
  for (int i = tid; i < D; i += kThreads) {
    float v = gstate[2 + i] * cM;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wstate[w * (D + 4)];
      if (mw != -INFINITY) v = fmaf(wstate[w * (D + 4) + 2 + i], __expf(mw - MM), v);
      v = fmaf(dstate[w * (D + 4) + 2 + i], cM, v);
    }
    out[i] = Elem<T>::from_f(v / L);
  }
  if (tid == 0 && a.lse) a.lse[orow] = MM + __logf(L);
  if (a.sel_groups)
    for (int i = tid; i < a.G; i += kThreads) a.sel_groups[orow * a.G + i] = i < nwin ? win[i].id : -1;
  if (a.sel_pages)
    for (int i = nwin * a.TP + tid; i < a.G * a.TP; i += kThreads) a.sel_pages[orow * a.G * a.TP + i] = -1;
}

template <typename T, int D, int NQ, int KG>
cudaError_t launch_t(const AttendArgs& a, cudaStream_t stream) {
  const int nsplit = a.nsg + a.nsw;
  const int64_t npos = a.seq_lens ? 1 : a.pos_hi - a.pos_lo;
  const int64_t rows = (int64_t)a.B * a.Hq * npos;
  cudaError_t e;
  if (a.units > 0 && nsplit > 0) {
    auto sk = scan_kernel<T, D, NQ, KG>;
    const size_t smem = ScanSmem<T, D, NQ>::bytes;
    e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sk<<<dim3((unsigned)a.units, (unsigned)nsplit), kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (rows > 0) {
    auto rk = refine_kernel<T, D, NQ, KG>;
    const size_t smem = RefineSmem<T, D>::bytes;
    e = cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, rk, a);
  }
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <typename T, int D, int NQ>
cudaError_t launch_kg(const AttendArgs& a, cudaStream_t stream) {
  return a.G <= 8 ? launch_t<T, D, NQ, 8>(a, stream) : launch_t<T, D, NQ, 16>(a, stream);
}

template <typename T, int D>
cudaError_t launch_nq(const AttendArgs& a, int NQ, cudaStream_t stream) {
  switch (NQ) {
    case 1: return launch_kg<T, D, 1>(a, stream);
    case 2: return launch_kg<T, D, 2>(a, stream);
    case 4: return launch_kg<T, D, 4>(a, stream);
    case 8: return launch_kg<T, D, 8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t cand_bytes() { return sizeof(Cand); }

cudaError_t launch_attend(const AttendArgs& a, int dtype, int d, int NQ, cudaStream_t stream) {
  if (dtype == LOD_DTYPE_F32)
    return d == 64 ? launch_nq<float, 64>(a, NQ, stream) : launch_nq<float, 128>(a, NQ, stream);
  return d == 64 ? launch_nq<__nv_bfloat16, 64>(a, NQ, stream)
                 : launch_nq<__nv_bfloat16, 128>(a, NQ, stream);
}

}  // namespace lod
