// lod_attend.cu -- LoD decode and prefill attention ("Level of Detail
// Attention", How It Works, paragraphs 2-3).
//
// Two kernels per batch of query rows:
//
//  scan    grid (unit, split).  A split streams either a slice of the unit's
//          visible group summaries (mean key, mean value, count) or a slice of
//          the exact window (plus the sinks).  Every row enters an online
//          softmax with logit scale*q.k + ln(count) (count 1 for exact
//          tokens), so the split leaves a partial state (max, sum, acc[d])
//          over ALL its rows; group splits also keep their local top-KG
//          groups by score scale*q.k (no count term).
//  refine  one CTA per query row.  It merges the split states, picks the
//          global top `top_groups` groups from the local candidates, and
//          removes those groups' coarse terms from the merged state (they are
//          about to be replaced by finer entries).  For each opened group it
//          scores the page summaries, opens the top `top_pages` pages and
//          adds their tokens exactly, adds the other pages as coarse entries
//          (page mean logit + ln(count), page mean value), and writes
//          out = acc / sum and the log-sum-exp.
//
// Removing the opened groups after the fact (instead of holding them out of
// the scan) is numerically safe: the terms that replace an opened group --
// its pages, or their tokens -- carry at least the group's own mass (the
// method's "conservative estimate" property: n exp(q.mean k) <= sum exp(q.k)),
// so the final normaliser is never smaller than what was subtracted and the
// cancellation error stays at the fp32 rounding level of the output.
#include "lod_internal.cuh"

namespace lod {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

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
  float s = 0.f;
#pragma unroll
  for (int v = 0; v < D / VEC; ++v) {
    float f[VEC];
    unpack16<T>(raw[v], f);
#pragma unroll
    for (int e = 0; e < VEC; ++e) s = fmaf(qs[v * VEC + e], f[e], s);
  }
  return s;
}

// Add a batch of up to 32 softmax entries (lane e: logit le, value row ve) to
// a warp's online-softmax state (m, l replicated; acc: the lane's DPL dims).
template <typename T, int D>
__device__ __forceinline__ void warp_add_entries(float le, const T* ve, bool valid, float& m, float& l,
                                                 float (&acc)[D / 32]) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const float bm = warp_max(valid ? le : -INFINITY);
  if (bm == -INFINITY) return;
  const float mn = fmaxf(m, bm);
  const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
  const float p = valid ? __expf(le - mn) : 0.f;
  l = l * corr + warp_sum(p);
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] *= corr;
  m = mn;
  const unsigned vm = __ballot_sync(0xffffffffu, valid);
  const uintptr_t vp = reinterpret_cast<uintptr_t>(ve);
  // coalesced value rows: all lanes read row e, DPL dims each
  for (int base = 0; base < 32; base += 8) {
    if (!((vm >> base) & 0xffu)) continue;
    float vv[8][DPL];
    float pe[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = base + j;
      pe[j] = __shfl_sync(0xffffffffu, p, e);
      const uintptr_t rp = __shfl_sync(0xffffffffu, (unsigned long long)vp, e);
      if ((vm >> e) & 1u) {
        load_f<T, DPL>(reinterpret_cast<const T*>(rp) + lane * DPL, vv[j]);
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) vv[j][i] = 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pe[j], vv[j][i], acc[i]);
  }
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

// ------------------------------------------------------------------ scan

template <typename T, int D, int NQ, int KG>
__global__ void __launch_bounds__(kThreads) scan_kernel(AttendArgs a) {
  constexpr int DPL = D / 32;
  const int64_t u = blockIdx.x;
  const int s = blockIdx.y;
  const int nsplit = a.nsg + a.nsw;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const UnitInfo ui = unit_info(a, u);

  extern __shared__ __align__(16) float sm[];
  float* st_s = sm;                                          // [kWarps][NQ][D+2]
  float* cs_s = st_s + kWarps * NQ * (D + 2);                // [kWarps][NQ][KG]
  int* ci_s = reinterpret_cast<int*>(cs_s + kWarps * NQ * KG);

  // rows of this unit: positions and validity
  int64_t t_row[NQ];
  bool ok[NQ];
  int64_t t_max = -1;
  bool bad_len = false;
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    if (a.seq_lens) {
      const int64_t L = a.seq_lens[ui.b];
      ok[r] = (r < a.g) && L >= 1 && L <= a.Tmax;
      bad_len = !(L >= 1 && L <= a.Tmax);
      t_row[r] = L - 1;
    } else {
      const int64_t pi = a.pos_lo + ui.blk * a.NP + r / a.g;
      ok[r] = (r < a.g * a.NP) && pi < a.pos_hi;
      t_row[r] = a.q_begin + pi;
    }
    if (ok[r] && t_row[r] > t_max) t_max = t_row[r];
  }
  if (bad_len && s == 0 && threadIdx.x == 0) set_status(a.status, LOD_ST_BAD_SEQLEN);

  // query rows (pre-scaled), this lane's DPL dims
  float qf[NQ][DPL];
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    if (ok[r]) {
      const int hq = ui.kvh * a.g + (r % a.g);
      const int64_t pi = a.seq_lens ? 0 : a.pos_lo + ui.blk * a.NP + r / a.g;
      const T* qp = static_cast<const T*>(a.q) + (((int64_t)ui.b * a.Hq + hq) * a.Tq + pi) * D;
      load_f<T, DPL>(qp + lane * DPL, qf[r]);
#pragma unroll
      for (int i = 0; i < DPL; ++i) qf[r][i] *= a.scale;
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) qf[r][i] = 0.f;
    }
  }

  float m[NQ], l[NQ], acc[NQ][DPL];
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[r][i] = 0.f;
  }
  bool myok = false;  // lane r < NQ owns row r's candidate list
#pragma unroll
  for (int r = 0; r < NQ; ++r)
    if (lane == r) myok = ok[r];
  float cs[KG];
  int ci[KG];
#pragma unroll
  for (int j = 0; j < KG; ++j) {
    cs[j] = -INFINITY;
    ci[j] = -1;
  }

  if (t_max >= 0) {
    const int64_t bt = t_max / kChunk;
    const int64_t nw = a.window / kChunk;
    const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;  // visible chunks [0, wb)
    const int64_t ws = wb * kChunk;                          // window start
    const int64_t unit_kv = (int64_t)ui.b * a.Hkv + ui.kvh;
    const T* Kb = static_cast<const T*>(a.K) + ui.b * a.sb + ui.kvh * a.sh;
    const T* Vb = static_cast<const T*>(a.V) + ui.b * a.sb + ui.kvh * a.sh;

    if (s < a.nsg) {
      // ---- a slice of the visible group summaries
      const int64_t G_vis = wb * a.k;
      const int64_t lo = (int64_t)s * kScanRows;
      const int64_t hi = lo + kScanRows < G_vis ? lo + kScanRows : G_vis;
      const T* gK = static_cast<const T*>(a.gK) + unit_kv * a.Cmax * a.k * D;
      const T* gV = static_cast<const T*>(a.gV) + unit_kv * a.Cmax * a.k * D;
      const int32_t* gC = a.gCnt + unit_kv * a.Cmax * a.k;
      for (int64_t gid = lo + warp; gid < hi; gid += kWarps) {
        const int cnt = gC[gid];
        if (cnt <= 0) continue;  // empty group slot
        if (cnt > kChunk) {
          if (lane == 0) set_status(a.status, LOD_ST_BAD_COUNT);
          continue;
        }
        float kf[DPL], vf[DPL];
        load_f<T, DPL>(gK + gid * D + lane * DPL, kf);
        load_f<T, DPL>(gV + gid * D + lane * DPL, vf);
        const float lnc = __logf((float)cnt);
        float sc[NQ];
#pragma unroll
        for (int r = 0; r < NQ; ++r) {
          float p = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) p = fmaf(qf[r][i], kf[i], p);
          sc[r] = warp_sum(p);
        }
        float mine = -INFINITY;
#pragma unroll
        for (int r = 0; r < NQ; ++r) {
          if (!ok[r]) continue;
          if (lane == r) mine = sc[r];
          const float lg = sc[r] + lnc;
          if (lg > m[r]) {
            const float corr = __expf(m[r] - lg);
            l[r] *= corr;
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[r][i] *= corr;
            m[r] = lg;
          }
          const float p = __expf(lg - m[r]);
          l[r] += p;
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[r][i] = fmaf(p, vf[i], acc[r][i]);
        }
        // lane r keeps row r's local top-KG (score desc, id asc)
        if (myok && cand_better(mine, (int)gid, cs[KG - 1], ci[KG - 1])) {
          float ns = mine;
          int ni = (int)gid;
#pragma unroll
          for (int j = 0; j < KG; ++j) {
            if (cand_better(ns, ni, cs[j], ci[j])) {
              const float ts = cs[j];
              const int ti = ci[j];
              cs[j] = ns;
              ci[j] = ni;
              ns = ts;
              ni = ti;
            }
          }
        }
      }
    } else {
      // ---- a slice of the exact window; slice 0 also takes the sinks
      const int64_t wi = s - a.nsg;
      const int64_t lo = ws + wi * kScanRows;
      const int64_t hi = lo + kScanRows < t_max + 1 ? lo + kScanRows : t_max + 1;
      const int64_t ns = wi == 0 ? (a.sinks < ws ? a.sinks : ws) : 0;
      const int64_t nrows = (hi > lo ? hi - lo : 0) + ns;
      for (int64_t e = warp; e < nrows; e += kWarps) {
        const int64_t pos = e < ns ? e : lo + (e - ns);
        float kf[DPL], vf[DPL];
        load_f<T, DPL>(Kb + pos * a.st + lane * DPL, kf);
        load_f<T, DPL>(Vb + pos * a.st + lane * DPL, vf);
#pragma unroll
        for (int r = 0; r < NQ; ++r) {
          float p = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) p = fmaf(qf[r][i], kf[i], p);
          const float lg = warp_sum(p);
          if (!ok[r] || pos > t_row[r]) continue;  // causal mask within the window
          if (lg > m[r]) {
            const float corr = __expf(m[r] - lg);
            l[r] *= corr;
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[r][i] *= corr;
            m[r] = lg;
          }
          const float pe = __expf(lg - m[r]);
          l[r] += pe;
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[r][i] = fmaf(pe, vf[i], acc[r][i]);
        }
      }
    }
  }

  // ---- combine the warps' states and candidates
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    float* dst = st_s + (warp * NQ + r) * (D + 2);
    if (lane == 0) {
      dst[0] = m[r];
      dst[1] = l[r];
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[2 + lane * DPL + i] = acc[r][i];
  }
  if (lane < NQ) {
#pragma unroll
    for (int j = 0; j < KG; ++j) {
      cs_s[(warp * NQ + lane) * KG + j] = cs[j];
      ci_s[(warp * NQ + lane) * KG + j] = ci[j];
    }
  }
  __syncthreads();
  float* part = a.part + ((u * nsplit + s) * NQ) * (int64_t)(D + 2);
  for (int idx = threadIdx.x; idx < NQ * (D + 2); idx += kThreads) {
    const int r = idx / (D + 2), c = idx % (D + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, st_s[(w * NQ + r) * (D + 2)]);
    float v;
    if (c == 0) {
      v = M;
    } else {
      v = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float mw = st_s[(w * NQ + r) * (D + 2)];
          if (mw != -INFINITY) v = fmaf(st_s[(w * NQ + r) * (D + 2) + c], __expf(mw - M), v);
        }
      }
    }
    part[idx] = v;
  }
  if (s < a.nsg) {
    // per row: best KG of the kWarps * KG warp candidates
    for (int r = warp; r < NQ; r += kWarps) {
      float c0[kWarps * KG / 32 > 0 ? kWarps * KG / 32 : 1];
      int i0[kWarps * KG / 32 > 0 ? kWarps * KG / 32 : 1];
      constexpr int PER = kWarps * KG / 32;
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = lane + 32 * j;
        const int w = e / KG, jj = e % KG;
        c0[j] = cs_s[(w * NQ + r) * KG + jj];
        i0[j] = ci_s[(w * NQ + r) * KG + jj];
      }
      float* cso = a.cand_s + ((u * a.nsg + s) * NQ + r) * (int64_t)KG;
      int* cio = a.cand_i + ((u * a.nsg + s) * NQ + r) * (int64_t)KG;
      for (int rank = 0; rank < KG; ++rank) {
        float bs = -INFINITY;
        int bi = -1;
#pragma unroll
        for (int j = 0; j < PER; ++j)
          if (i0[j] >= 0 && (bi < 0 || cand_better(c0[j], i0[j], bs, bi))) {
            bs = c0[j];
            bi = i0[j];
          }
        // empty lanes carry (-inf, INT_MAX), which loses to every real candidate
        float win_s = bi < 0 ? -INFINITY : bs;
        int win_i = bi < 0 ? 0x7fffffff : bi;
        warp_best(win_s, win_i);
        if (lane == 0) {
          cso[rank] = win_s;
          cio[rank] = (win_i == 0x7fffffff) ? -1 : win_i;
        }
#pragma unroll
        for (int j = 0; j < PER; ++j)
          if (i0[j] == win_i) i0[j] = -1;  // remove the winner (ids are unique)
      }
    }
  }
}

// ------------------------------------------------------------------ refine

template <typename T, int D, int NQ, int KG>
__global__ void __launch_bounds__(kThreads) refine_kernel(AttendArgs a) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nsplit = a.nsg + a.nsw;
  const int64_t npos = a.seq_lens ? 1 : a.pos_hi - a.pos_lo;
  const int64_t row = blockIdx.x;
  const int b = (int)(row / (a.Hq * npos));
  const int hq = (int)((row / npos) % a.Hq);
  const int64_t pi = a.seq_lens ? 0 : a.pos_lo + row % npos;
  const int kvh = hq / a.g, hh = hq % a.g;
  int64_t u;
  int r;
  int64_t t;
  if (a.seq_lens) {
    u = (int64_t)b * a.Hkv + kvh;
    r = hh;
    t = a.seq_lens[b] - 1;
  } else {
    const int64_t nblk = (a.pos_hi - a.pos_lo + a.NP - 1) / a.NP;
    const int64_t rel = pi - a.pos_lo;
    u = ((int64_t)b * a.Hkv + kvh) * nblk + rel / a.NP;
    r = (int)(rel % a.NP) * a.g + hh;
    t = a.q_begin + pi;
  }
  const int64_t orow = ((int64_t)b * a.Hq + hq) * a.Tq + pi;  // row of q / out / lse
  T* out = static_cast<T*>(a.out) + orow * D;

  __shared__ float qs[D];
  __shared__ float gstate[D + 2];
  __shared__ float wstate[kWarps][D + 2];
  __shared__ float win_s[kMaxTopGroups];
  __shared__ int win_i[kMaxTopGroups];
  __shared__ int nwin_s;

  if (t < 0 || t >= a.Tmax) {  // invalid sequence length (decode)
    for (int i = threadIdx.x; i < D; i += kThreads) out[i] = Elem<T>::from_f(0.f);
    if (threadIdx.x == 0) {
      set_status(a.status, LOD_ST_BAD_SEQLEN);
      if (a.lse) a.lse[orow] = -INFINITY;
    }
    if (a.sel_groups)
      for (int i = threadIdx.x; i < a.G; i += kThreads) a.sel_groups[orow * a.G + i] = -1;
    if (a.sel_pages)
      for (int i = threadIdx.x; i < a.G * a.TP; i += kThreads) a.sel_pages[orow * a.G * a.TP + i] = -1;
    return;
  }

  const T* qp = static_cast<const T*>(a.q) + orow * D;
  for (int i = threadIdx.x; i < D; i += kThreads) qs[i] = Elem<T>::to_f(qp[i]) * a.scale;

  // ---- global top-G over the group splits' candidates (warp 0)
  if (warp == 0) {
    const int ncand = a.nsg * KG;
    const float* csrc = a.cand_s + (u * a.nsg * NQ) * (int64_t)KG;
    const int* isrc = a.cand_i + (u * a.nsg * NQ) * (int64_t)KG;
    float lastS = INFINITY;
    int lastI = -1;
    int nwin = 0;
    for (int rank = 0; rank < a.G; ++rank) {
      // best candidate strictly worse than the previous winner
      float bs = -INFINITY;
      int bi = 0x7fffffff;
      for (int e = lane; e < ncand; e += 32) {
        const int sp = e / KG, j = e % KG;
        const int64_t off = ((int64_t)sp * NQ + r) * KG + j;
        const int id = isrc[off];
        if (id < 0) continue;
        const float sc = csrc[off];
        const bool after = rank == 0 || cand_better(lastS, lastI, sc, id);
        if (after && (bi == 0x7fffffff || cand_better(sc, id, bs, bi))) {
          bs = sc;
          bi = id;
        }
      }
      warp_best(bs, bi);
      if (bi == 0x7fffffff) break;
      if (lane == 0) {
        win_s[rank] = bs;
        win_i[rank] = bi;
      }
      lastS = bs;
      lastI = bi;
      ++nwin;
    }
    if (lane == 0) nwin_s = nwin;
  }

  // ---- merge the split states (thread c owns component c: m, l, acc[])
  {
    const float* ps = a.part + (u * nsplit * NQ + r) * (int64_t)(D + 2);
    const int64_t stride = (int64_t)NQ * (D + 2);
    float M = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, ps[sp * stride]);
    for (int c = threadIdx.x; c < D + 2; c += kThreads) {
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
  const int nwin = nwin_s;
  const float M = gstate[0];
  const int64_t unit_kv = (int64_t)b * a.Hkv + kvh;

  // ---- take the opened groups' coarse terms back out
  {
    const T* gV = static_cast<const T*>(a.gV) + unit_kv * a.Cmax * a.k * D;
    const int32_t* gC = a.gCnt + unit_kv * a.Cmax * a.k;
    for (int c = threadIdx.x; c < D + 1; c += kThreads) {
      float v = gstate[c + 1];
      for (int w = 0; w < nwin; ++w) {
        const int id = win_i[w];
        const float e = __expf(win_s[w] + __logf((float)gC[id]) - M);
        v -= e * (c == 0 ? 1.f : Elem<T>::to_f(gV[(int64_t)id * D + (c - 1)]));
      }
      gstate[c + 1] = v;
    }
  }

  // ---- pages of the opened groups: warp w handles opened groups w, w+8, ...
  float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  const T* pK = static_cast<const T*>(a.pK) + unit_kv * a.Cmax * a.P * D;
  const T* pV = static_cast<const T*>(a.pV) + unit_kv * a.Cmax * a.P * D;
  const int32_t* pC = a.pCnt + unit_kv * a.Cmax * a.P;
  const int16_t* pB = a.pBeg + unit_kv * a.Cmax * a.P;
  const int16_t* gP = a.gPage + unit_kv * a.Cmax * (a.k + 1);
  const int16_t* pm = a.perm + unit_kv * a.Cmax * kChunk;
  const T* Kb = static_cast<const T*>(a.K) + b * a.sb + kvh * a.sh;
  const T* Vb = static_cast<const T*>(a.V) + b * a.sb + kvh * a.sh;
  for (int w = warp; w < nwin; w += kWarps) {
    const int id = win_i[w];
    const int64_t c = id / a.k;
    const int j = id % a.k;
    const int p0 = gP[c * (a.k + 1) + j], p1 = gP[c * (a.k + 1) + j + 1];
    int open_slot[kMaxTopPages];
#pragma unroll
    for (int x = 0; x < kMaxTopPages; ++x) open_slot[x] = -1;
    if (p0 < 0 || p1 < p0 || p1 > a.P || p1 - p0 > 32) {
      if (lane == 0) set_status(a.status, LOD_ST_BAD_PAGE);
    } else {
      const int np = p1 - p0;
      // lane p scores page p0 + p
      float sc = -INFINITY;
      int cntp = 0;
      if (lane < np) {
        cntp = pC[c * a.P + p0 + lane];
        sc = row_dot<T, D>(pK + (c * a.P + p0 + lane) * D, qs);
      }
      // top-TP pages by (score desc, slot asc)
      float s2 = sc;
      int sl2 = lane < np ? p0 + lane : 0x7fffffff;
      int nopen = 0;
      for (int x = 0; x < a.TP && x < np; ++x) {
        float bs = s2;
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
      // coarse entries: unopened pages
      const bool cvalid = lane < np && !is_open && cntp > 0 && cntp <= kPage;
      if (lane < np && !is_open && (cntp <= 0 || cntp > kPage)) set_status(a.status, LOD_ST_BAD_COUNT);
      warp_add_entries<T, D>(cvalid ? sc + __logf((float)cntp) : -INFINITY,
                             pV + (c * a.P + p0 + (lane < np ? lane : 0)) * D, cvalid, m, l, acc);
      // exact entries: members of the opened pages, one lane per member
      for (int x = 0; x < nopen; ++x) {
        const int slot = open_slot[x];
        const int beg = pB[c * a.P + slot];
        const int n = pC[c * a.P + slot];
        bool okp = beg >= 0 && n > 0 && n <= kPage && beg + n <= kChunk;
        if (!okp && lane == 0) set_status(a.status, LOD_ST_BAD_PAGE);
        bool ev = okp && lane < n;
        int off = ev ? pm[c * kChunk + beg + lane] : 0;
        if (ev && (off < 0 || off >= kChunk)) {
          set_status(a.status, LOD_ST_BAD_MEMBER);
          ev = false;
        }
        const int64_t pos = c * kChunk + off;
        const float lg = ev ? row_dot<T, D>(Kb + pos * a.st, qs) : -INFINITY;
        warp_add_entries<T, D>(lg, Vb + pos * a.st, ev, m, l, acc);
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
  // ---- final merge: per-warp page states + the group/window state
  if (lane == 0) {
    wstate[warp][0] = m;
    wstate[warp][1] = l;
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i) wstate[warp][2 + lane * DPL + i] = acc[i];
  __syncthreads();
  float MM = M;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) MM = fmaxf(MM, wstate[w][0]);
  float L = gstate[1] * __expf(M - MM);
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (wstate[w][0] != -INFINITY) L = fmaf(wstate[w][1], __expf(wstate[w][0] - MM), L);
  for (int i = threadIdx.x; i < D; i += kThreads) {
    float v = gstate[2 + i] * __expf(M - MM);
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (wstate[w][0] != -INFINITY) v = fmaf(wstate[w][2 + i], __expf(wstate[w][0] - MM), v);
    out[i] = Elem<T>::from_f(v / L);
  }
  if (threadIdx.x == 0 && a.lse) a.lse[orow] = MM + __logf(L);
  if (a.sel_groups)
    for (int i = threadIdx.x; i < a.G; i += kThreads)
      a.sel_groups[orow * a.G + i] = i < nwin ? win_i[i] : -1;
  if (a.sel_pages)
    for (int i = nwin * a.TP + threadIdx.x; i < a.G * a.TP; i += kThreads)
      a.sel_pages[orow * a.G * a.TP + i] = -1;
}

template <typename T, int D, int NQ, int KG>
cudaError_t launch_t(const AttendArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(float) * kWarps * NQ * (D + 2) + (sizeof(float) + sizeof(int)) * kWarps * NQ * KG;
  auto sk = scan_kernel<T, D, NQ, KG>;
  cudaError_t e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nsplit = a.nsg + a.nsw;
  if (a.units > 0 && nsplit > 0) {
    sk<<<dim3((unsigned)a.units, (unsigned)nsplit), kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t npos = a.seq_lens ? 1 : a.pos_hi - a.pos_lo;
  const int64_t rows = (int64_t)a.B * a.Hq * npos;
  if (rows > 0) {
    refine_kernel<T, D, NQ, KG><<<(unsigned)rows, kThreads, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  return e;
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
    default:
      if constexpr (D == 64) return launch_kg<T, D, 16>(a, stream);
      return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_attend(const AttendArgs& a, int dtype, int d, int NQ, cudaStream_t stream) {
  if (dtype == LOD_DTYPE_F32)
    return d == 64 ? launch_nq<float, 64>(a, NQ, stream) : launch_nq<float, 128>(a, NQ, stream);
  return d == 64 ? launch_nq<__nv_bfloat16, 64>(a, NQ, stream)
                 : launch_nq<__nv_bfloat16, 128>(a, NQ, stream);
}

}  // namespace lod
