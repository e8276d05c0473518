// lod_build.cu -- online multi-resolution index build ("Level of Detail
// Attention", How It Works, paragraph 1): per 256-token chunk, k-means groups,
// 16-key pages, and their mean keys, mean values and counts.
//
// One CTA of 256 threads per (chunk, KV head, sequence).
// The chunk's keys are staged in shared memory by one TMA bulk copy; thread i
// also keeps key i in registers in the cache's packed form.  Centroids live
// in shared memory as fp32 pairs, interleaved by cluster, and are read as
// warp-uniform (broadcast) loads, so the assignment step is one packed fp32x2
// FMA per (key, centroid, two dimensions) in the expanded form
// ||c||^2 - 2 k.c (the ||k||^2 term is common to all centroids of a key).
//
// The update step is deterministic: members are counting-sorted by cluster
// (stable, ascending position) and every (cluster, dimension) sum is taken in
// a fixed order.  An iteration whose assignment equals the previous one
// therefore reproduces the previous centroids bit for bit, every later round
// would repeat it, and the loop stops there with an unchanged result.
//
// Summaries: each warp sums whole pages (its V rows read with coalesced
// loads, all in flight), writes the page means and keeps the page sums in
// shared memory; a group's mean value is the sum of its pages' sums, and its
// mean key is the final centroid.
#include "lod_internal.cuh"

namespace lod {

namespace {

constexpr int kBuildThreads = 256;
constexpr int kBuildWarps = kBuildThreads / 32;

template <int NW>
__device__ __forceinline__ void block_argmax(float v, int idx, float* red_s, int* red_i, float& out_v,
                                             int& out_i) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // larger value first, ties to the lower index
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
    if (v2 > v || (v2 == v && i2 < idx)) {
      v = v2;
      idx = i2;
    }
  }
  if (lane == 0) {
    red_s[warp] = v;
    red_i[warp] = idx;
  }
  __syncthreads();
  if (warp == 0) {
    v = lane < NW ? red_s[lane] : -INFINITY;
    idx = lane < NW ? red_i[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
      if (v2 > v || (v2 == v && i2 < idx)) {
        v = v2;
        idx = i2;
      }
    }
    if (lane == 0) {
      red_s[NW] = v;
      red_i[NW] = idx;
    }
  }
  __syncthreads();
  out_v = red_s[NW];
  out_i = red_i[NW];
  __syncthreads();
}

// Element pair p (dims 2p, 2p+1) of a key held as packed 32-bit words.
template <typename T>
__device__ __forceinline__ float2 pair_of(const uint32_t* w, int p) {
  if constexpr (sizeof(T) == 2) {
    return make_float2(__uint_as_float(w[p] << 16), __uint_as_float(w[p] & 0xffff0000u));
  } else {
    return make_float2(__uint_as_float(w[2 * p]), __uint_as_float(w[2 * p + 1]));
  }
}

// Three-tier INT4 ("Level of Detail Attention", the paragraph after the
// quality tables: INT4 KV storage, only the selected pages decompressed):
// one page's members as 4-bit codes of a per-channel asymmetric quantiser.
// Lane `lane` owns channels [lane * DPL, lane * DPL + DPL); get(r, i) is
// member r's value in the lane's channel i.  Per channel: low = min, scale =
// (max - low) / 15, code = clamp(rint((x - low) / scale), 0, 15) (0 when
// scale = 0), all in IEEE fp32.  codes: the page's first member-ordered row
// (d/2 bytes per row, channel 2i in the low nibble); qs: (scale, low) per
// channel of the page slot.
template <int D, int DPL, typename Get>
__device__ __forceinline__ void quantize_page(int pc, Get get, uint8_t* codes, float2* qs, int lane) {
  float lo[DPL], sc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < kPage; ++r) {
      if (r < pc) {
        const float x = get(r, i);
        if (x < mn) mn = x;
        if (x > mx) mx = x;
      }
    }
    lo[i] = mn;
    sc[i] = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    qs[lane * DPL + i] = make_float2(sc[i], lo[i]);
  }
#pragma unroll
  for (int r = 0; r < kPage; ++r) {
    if (r >= pc) break;
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      float v = sc[i] > 0.0f ? rintf(__fdiv_rn(__fsub_rn(get(r, i), lo[i]), sc[i])) : 0.0f;
      v = fminf(fmaxf(v, 0.0f), 15.0f);
      w |= (uint32_t)v << (4 * i);
    }
    uint8_t* dst = codes + (int64_t)r * (D / 2) + lane * (DPL / 2);
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint16_t*>(dst) = (uint16_t)w;
    } else {
      static_assert(DPL == 2, "channels per lane");
      *dst = (uint8_t)w;
    }
  }
}

template <typename T, int D, int KMAX>
struct BuildSmem {
  static constexpr int PMAX = kChunk / kPage + KMAX;  // page slots per chunk
  static constexpr size_t off_x = 0;                                        // T [256][D]
  static constexpr size_t off_cen = (size_t)kChunk * D * sizeof(T);         // float2 [D/2][KMAX]
  static constexpr size_t off_psum = off_cen + sizeof(float) * D * KMAX;    // float [PMAX][D] value sums
  static constexpr size_t off_cn = off_psum + sizeof(float) * PMAX * D;     // float [KMAX][D/64] norm parts
  static constexpr size_t off_red = off_cn + sizeof(float) * KMAX * (D / 64);  // float/int [NW+1] x 2
  static constexpr size_t off_wc = off_red + 8 * (kBuildWarps + 1);         // int [NW][KMAX]
  static constexpr size_t off_cnt = off_wc + 4 * kBuildWarps * KMAX;        // int [KMAX]
  static constexpr size_t off_off = off_cnt + 4 * KMAX;                     // int [KMAX+1]
  static constexpr size_t off_ps = off_off + 4 * (KMAX + 1);                // int [KMAX+1]
  static constexpr size_t off_perm = off_ps + 4 * (KMAX + 1);               // int [256]
  static constexpr size_t off_bar = (off_perm + 4 * kChunk + 7) & ~size_t(7);
  static constexpr size_t bytes = off_bar + 8;
};

// Two CTAs per SM where the packed key (up to 256 bytes, with up to 8
// clusters; any count for 128-byte keys) fits in half the register file;
// one otherwise.
template <typename T, int D, int KMAX>
__global__ void __launch_bounds__(kBuildThreads,
                                  (D * sizeof(T) <= 128 || (D * sizeof(T) <= 256 && KMAX <= 8)) ? 2 : 1)
    kmeans_kernel(BuildArgs a) {
  constexpr int NW = kBuildWarps;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int NWORD = D * (int)sizeof(T) / 4;  // packed 32-bit words per key
  constexpr int NP = D / 2;                      // dimension pairs
  using SM = BuildSmem<T, D, KMAX>;
  constexpr int PMAX = SM::PMAX;
  const int h = blockIdx.y, b = blockIdx.z;
  int64_t cc = a.chunk_begin + blockIdx.x;
  if (a.seq_lens) {  // online build: the chunk sequence b's length has just completed, if any
    const int64_t L = a.seq_lens[b];
    if (L < kChunk || L % kChunk != 0 || L / kChunk > a.Cmax) return;
    cc = L / kChunk - 1;
  }
  const int64_t c = cc;
  const int64_t unit = (int64_t)b * a.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int first = (c == 0) ? a.sinks : 0;  // sink positions are never clustered
  const int n = kChunk - first;
  const int k = a.k;

  extern __shared__ __align__(128) unsigned char smem[];
  T* xs = reinterpret_cast<T*>(smem + SM::off_x);
  float2* cen2 = reinterpret_cast<float2*>(smem + SM::off_cen);
  float* psum = reinterpret_cast<float*>(smem + SM::off_psum);
  float* cnorm = reinterpret_cast<float*>(smem + SM::off_cn);
  float* red_s = reinterpret_cast<float*>(smem + SM::off_red);
  int* red_i = reinterpret_cast<int*>(red_s + NW + 1);
  int* wcnt = reinterpret_cast<int*>(smem + SM::off_wc);
  int* cnt = reinterpret_cast<int*>(smem + SM::off_cnt);
  int* off = reinterpret_cast<int*>(smem + SM::off_off);
  int* pstart = reinterpret_cast<int*>(smem + SM::off_ps);
  int* perm_s = reinterpret_cast<int*>(smem + SM::off_perm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM::off_bar);

  const T* Kc = static_cast<const T*>(a.K) + b * a.sb + h * a.sh + c * kChunk * a.st;
  const T* Vc = static_cast<const T*>(a.V) + b * a.sb + h * a.sh + c * kChunk * a.st;

  // ---- stage the chunk's keys in shared memory (TMA) and own key in registers
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect(bar, (uint32_t)kChunk * ROWB);
    __syncwarp();
    if (a.st == D) {
      if (lane == 0) bulk_g2s(xs, Kc, (uint32_t)kChunk * ROWB, bar);
    } else {
      for (int r = lane; r < kChunk; r += 32) bulk_g2s(xs + r * D, Kc + (int64_t)r * a.st, ROWB, bar);
    }
  }
  uint32_t kw[NWORD];
  // Keeps the key packed: without it the compiler hoists the unpacked fp32
  // key (twice the registers) out of the rounds, which halves the occupancy.
  auto keep_packed = [&]() {
    if constexpr (ROWB == 256) {
#pragma unroll
      for (int w = 0; w < NWORD; ++w) asm volatile("" : "+r"(kw[w]));
    }
  };
  {
    const uint4* row = reinterpret_cast<const uint4*>(Kc + (int64_t)(tid < n ? first + tid : first) * a.st);
#pragma unroll
    for (int v = 0; v < NWORD / 4; ++v) {
      const uint4 r = __ldg(row + v);
      kw[4 * v] = r.x;
      kw[4 * v + 1] = r.y;
      kw[4 * v + 2] = r.z;
      kw[4 * v + 3] = r.w;
    }
  }
  const bool staged = mbar_wait(bar, 0, a.status);
  if (!__syncthreads_and(staged)) {  // copy timed out: leave this chunk unwritten
    if (tid == 0) (void)mbar_wait(bar, 0, a.status);
    return;
  }
  auto xval = [&](int row, int d) { return Elem<T>::to_f(xs[row * D + d]); };
  // dims 2p and 2p+1 of a staged key, one shared-memory load
  auto xpair = [&](int row, int p) {
    return pair_of<T>(reinterpret_cast<const uint32_t*>(xs + row * D), p);
  };

  // ---- seeded farthest-first initialisation
  float mind = tid < n ? INFINITY : -INFINITY;
  for (int j = 0; j < k; ++j) {
    keep_packed();
    int pick;
    if (j == 0) {
      // the initialisation's sequence-head index is model-wide under head sharding
      const int64_t sunit = a.head_shard ? (int64_t)b * (a.head_shard >> 16) + (a.head_shard & 0xffff) + h : unit;
      const uint64_t hsh = splitmix64(a.seed ^ ((uint64_t(sunit) << 32) + uint64_t(c)));
      pick = (int)(hsh % uint64_t(n));
    } else {
      float bv;
      block_argmax<NW>(tid < n ? mind : -INFINITY, tid, red_s, red_i, bv, pick);
    }
    for (int p = tid; p < NP; p += kBuildThreads)
      cen2[p * KMAX + j] = make_float2(xval(first + pick, 2 * p), xval(first + pick, 2 * p + 1));
    __syncthreads();
    if (tid < n) {
      float dd = 0.f;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 x = pair_of<T>(kw, p);
        const float2 cc = cen2[p * KMAX + j];
        const float t0 = x.x - cc.x, t1 = x.y - cc.y;
        dd = fmaf(t0, t0, dd);
        dd = fmaf(t1, t1, dd);
      }
      mind = fminf(mind, dd);
    }
  }
  // ||c_j||^2 in D/64 parts of 32 dimension pairs: item (j, p) = j * NP + p;
  // the 32 items of a warp belong to one cluster (NP is a multiple of 32)
  constexpr int NSLOT = NP / 32;
  static_assert(NP % 32 == 0, "dimension pairs per warp");
  auto norm_part = [&](int item, float2 cc) {
    const float s = warp_sum(fmaf(cc.x, cc.x, cc.y * cc.y));
    if (lane == 0) cnorm[item >> 5] = s;
  };
  for (int item = tid; item < k * NP; item += kBuildThreads)
    norm_part(item, cen2[(item % NP) * KMAX + item / NP]);
  __syncthreads();

  // ---- Lloyd rounds
  int a_prev = -1;
  for (int it = 0; it < a.iters; ++it) {
    keep_packed();
    int a_new = 0;
    if (tid < n) {
      float2 dot[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) dot[j] = make_float2(0.f, 0.f);
      if constexpr (KMAX <= 8) {
        // every slot of the centroid row, two per 16-byte load (the slots
        // past k hold no centroid; their sums are never read)
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const float2 x = pair_of<T>(kw, p);
          const float4* c4 = reinterpret_cast<const float4*>(cen2 + p * KMAX);
#pragma unroll
          for (int j2 = 0; j2 < KMAX / 2; ++j2) {
            const float4 cc = c4[j2];
            dot[2 * j2] = ffma2(x, make_float2(cc.x, cc.y), dot[2 * j2]);
            dot[2 * j2 + 1] = ffma2(x, make_float2(cc.z, cc.w), dot[2 * j2 + 1]);
          }
        }
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const float2 x = pair_of<T>(kw, p);
#pragma unroll
          for (int j = 0; j < KMAX; ++j)
            if (j < k) dot[j] = ffma2(x, cen2[p * KMAX + j], dot[j]);
        }
      }
      auto cn = [&](int j) {
        float v = cnorm[j * NSLOT];
#pragma unroll
        for (int t = 1; t < NSLOT; ++t) v += cnorm[j * NSLOT + t];
        return v;
      };
      float best = fmaf(-2.f, dot[0].x + dot[0].y, cn(0));
#pragma unroll
      for (int j = 1; j < KMAX; ++j) {
        if (j < k) {
          const float dj = fmaf(-2.f, dot[j].x + dot[j].y, cn(j));
          if (dj < best) {  // strict: ties keep the lower cluster id
            best = dj;
            a_new = j;
          }
        }
      }
    }
    // stable counting sort of members by cluster (ascending local index):
    // each warp's per-cluster counts, published by the change test's barrier
    int rank = 0;
    for (int j = 0; j < k; ++j) {
      const unsigned m = __ballot_sync(0xffffffffu, tid < n && a_new == j);
      if (lane == 0) wcnt[warp * KMAX + j] = __popc(m);
      if (tid < n && a_new == j) rank = __popc(m & ((1u << lane) - 1u));
    }
    const int changed = __syncthreads_or(tid < n && a_new != a_prev);
    if (it > 0 && !changed) break;  // fixed point: later rounds repeat this one exactly
    a_prev = a_new;
    {  // every thread takes its slot from the counts (cluster-major, then warp, then lane)
      int o = 0, slot = 0;
      for (int j = 0; j < k; ++j) {
        int cj = 0, before = 0;
        for (int w = 0; w < NW; ++w) {
          const int t = wcnt[w * KMAX + j];
          before += w < warp ? t : 0;
          cj += t;
        }
        if (j == a_new) slot = o + before + rank;
        if (tid == j) {
          off[j] = o;
          cnt[j] = cj;
        }
        o += cj;
      }
      if (tid == 0) off[k] = o;
      if (tid < n) perm_s[slot] = tid;
    }
    __syncthreads();

    // centroid := member mean (fp32, fixed order: four interleaved partial sums);
    // empty clusters keep theirs; then the centroid's norm parts
    for (int item = tid; item < k * NP; item += kBuildThreads) {
      const int j = item / NP, p = item % NP;
      const int cj = cnt[j];
      float2 cc = cen2[p * KMAX + j];
      if (cj > 0) {
        float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
        const int m0 = off[j], m1 = off[j] + cj;
        int m = m0;
        for (; m + 3 < m1; m += 4) {
          const float2 x0 = xpair(first + perm_s[m], p), x1 = xpair(first + perm_s[m + 1], p);
          const float2 x2 = xpair(first + perm_s[m + 2], p), x3 = xpair(first + perm_s[m + 3], p);
          s0.x += x0.x; s0.y += x0.y;
          s1.x += x1.x; s1.y += x1.y;
          s2.x += x2.x; s2.y += x2.y;
          s3.x += x3.x; s3.y += x3.y;
        }
        for (; m < m1; ++m) {
          const float2 x0 = xpair(first + perm_s[m], p);
          s0.x += x0.x;
          s0.y += x0.y;
        }
        const float sx = (s0.x + s1.x) + (s2.x + s3.x), sy = (s0.y + s1.y) + (s2.y + s3.y);
        cc = make_float2(sx / (float)cj, sy / (float)cj);
        cen2[p * KMAX + j] = cc;
      }
      norm_part(item, cc);
    }
    __syncthreads();
  }

  // ---- pages: group j's members in ascending position, runs of kPage
  if (tid == 0) {
    int s = 0;
    for (int j = 0; j < k; ++j) {
      pstart[j] = s;
      s += (cnt[j] + kPage - 1) / kPage;
    }
    pstart[k] = s;
  }
  __syncthreads();

  const int64_t P = a.P;
  T* gK = static_cast<T*>(a.gK) + (unit * a.Cmax * k + c * k) * D;
  T* gV = static_cast<T*>(a.gV) + (unit * a.Cmax * k + c * k) * D;
  T* pK = static_cast<T*>(a.pK) + (unit * a.Cmax * P + c * P) * D;
  T* pV = static_cast<T*>(a.pV) + (unit * a.Cmax * P + c * P) * D;
  int32_t* gCnt = a.gCnt + unit * a.Cmax * k + c * k;
  int32_t* pCnt = a.pCnt + unit * a.Cmax * P + c * P;
  int16_t* pBeg = a.pBeg + unit * a.Cmax * P + c * P;
  int16_t* gPage = a.gPage + unit * a.Cmax * (k + 1) + c * (k + 1);
  int16_t* perm = a.perm + unit * a.Cmax * kChunk + c * kChunk;

  perm[tid] = tid < n ? (int16_t)(first + perm_s[tid]) : (int16_t)-1;
  if (tid <= k) gPage[tid] = (int16_t)pstart[tid];
  if (tid < k) {
    gCnt[tid] = cnt[tid];
    a.gMeta[unit * a.Cmax * k + c * k + tid] = cnt[tid] | (pstart[tid] << 16) | (pstart[tid + 1] << 24);
  }
  const int used = pstart[k];
  if (tid < P) {
    if (tid < used) {
      int j = 0;
      while (j + 1 < k && pstart[j + 1] <= tid) ++j;
      const int pg = tid - pstart[j];
      pBeg[tid] = (int16_t)(off[j] + pg * kPage);
      pCnt[tid] = min(kPage, cnt[j] - pg * kPage);
    } else {
      pBeg[tid] = 0;
      pCnt[tid] = 0;
    }
  }

  // page sums: warp w takes pages w, w + NW, ...; lane owns DPL dims
  constexpr int DPL = D / 32;
  for (int pg = warp; pg < used; pg += NW) {
    int j = 0;
    while (j + 1 < k && pstart[j + 1] <= pg) ++j;
    const int m0 = off[j] + (pg - pstart[j]) * kPage;
    const int pc = min(kPage, cnt[j] - (pg - pstart[j]) * kPage);
    float vv[kPage][DPL];
#pragma unroll
    for (int r = 0; r < kPage; ++r) {
      if (r < pc) {
        load_f<T, DPL>(Vc + (int64_t)(first + perm_s[m0 + r]) * a.st + lane * DPL, vv[r]);
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) vv[r][i] = 0.f;
      }
    }
    float sk[DPL], sv[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) sk[i] = sv[i] = 0.f;
#pragma unroll
    for (int r = 0; r < kPage; ++r) {
      if (r < pc) {
        const int row = first + perm_s[m0 + r];
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          sk[i] += xval(row, lane * DPL + i);
          sv[i] += vv[r][i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      pK[pg * D + lane * DPL + i] = Elem<T>::from_f(sk[i] / (float)pc);
      pV[pg * D + lane * DPL + i] = Elem<T>::from_f(sv[i] / (float)pc);
      psum[pg * D + lane * DPL + i] = sv[i];
    }
    if (a.kv_bits == 4) {  // three-tier INT4: the page's members as 4-bit codes
      const int64_t mrow = (unit * a.Cmax + c) * kChunk + m0;  // member-ordered row of the first member
      const int64_t prow = (unit * a.Cmax + c) * P + pg;       // page slot
      quantize_page<D, DPL>(
          pc, [&](int r, int i) { return xval(first + perm_s[m0 + r], lane * DPL + i); },
          a.qK + mrow * (D / 2), a.qKs + prow * D, lane);
      quantize_page<D, DPL>(pc, [&](int r, int i) { return vv[r][i]; }, a.qV + mrow * (D / 2),
                            a.qVs + prow * D, lane);
    }
  }
  // member-ordered copies: row m = the token at chunk offset perm[m], so each
  // page's members are consecutive rows (keys from shared memory, values
  // from the rows the page sums just read); three-tier INT4 keeps codes instead
  if (a.kv_bits != 4) {
    constexpr int C16 = ROWB / 16;  // 16-byte pieces per row
    uint4* mKc = reinterpret_cast<uint4*>(static_cast<T*>(a.mK) + ((unit * a.Cmax + c) * kChunk) * D);
    uint4* mVc = reinterpret_cast<uint4*>(static_cast<T*>(a.mV) + ((unit * a.Cmax + c) * kChunk) * D);
    // four pieces per thread at a time, every load before any store (a
    // store would otherwise hold the next load back until the previous
    // load's round trip had ended)
    constexpr int U = 4;
    for (int base = tid; base < n * C16; base += U * kBuildThreads) {
      uint4 kq[U], vq[U];
#pragma unroll
      for (int x = 0; x < U; ++x) {
        const int item = base + x * kBuildThreads;
        if (item < n * C16) {
          const int m = item / C16, q = item % C16;
          const int row = first + perm_s[m];
          kq[x] = reinterpret_cast<const uint4*>(xs + row * D)[q];
          vq[x] = __ldg(reinterpret_cast<const uint4*>(Vc + (int64_t)row * a.st) + q);
        }
      }
#pragma unroll
      for (int x = 0; x < U; ++x) {
        const int item = base + x * kBuildThreads;
        if (item < n * C16) {
          mKc[item] = kq[x];
          mVc[item] = vq[x];
        }
      }
    }
  }
  // unused page slots hold zeros
  for (int item = tid; item < (int)(P - used) * D; item += kBuildThreads) {
    const int slot = used + item / D, i = item % D;
    pK[slot * D + i] = Elem<T>::from_f(0.f);
    pV[slot * D + i] = Elem<T>::from_f(0.f);
    if (a.kv_bits == 4) {
      const int64_t q = ((unit * a.Cmax + c) * P + slot) * D + i;
      a.qKs[q] = make_float2(0.f, 0.f);
      a.qVs[q] = make_float2(0.f, 0.f);
    }
  }
  __syncthreads();
  // group means: key = the final centroid; value = its pages' sums in page order
  for (int item = tid; item < k * D; item += kBuildThreads) {
    const int j = item / D, i = item % D;
    const int cj = cnt[j];
    if (cj == 0) {
      gK[j * D + i] = Elem<T>::from_f(0.f);
      gV[j * D + i] = Elem<T>::from_f(0.f);
      continue;
    }
    float s = 0.f;
    for (int pg = pstart[j]; pg < pstart[j + 1]; ++pg) s += psum[pg * D + i];
    const float2 cc = cen2[(i / 2) * KMAX + j];
    gK[j * D + i] = Elem<T>::from_f((i & 1) ? cc.y : cc.x);
    gV[j * D + i] = Elem<T>::from_f(s / (float)cj);
  }
  static_assert(PMAX >= kChunk / kPage, "page slots");
}

template <typename T, int D, int KMAX>
cudaError_t launch_kmeans_t(const BuildArgs& a, int64_t nchunks, int B, cudaStream_t stream) {
  const size_t smem = BuildSmem<T, D, KMAX>::bytes;
  auto kern = kmeans_kernel<T, D, KMAX>;
  cudaError_t e = set_smem_once<kmeans_kernel<T, D, KMAX>>(smem, true);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)nchunks, (unsigned)a.Hkv, (unsigned)B);
  kern<<<grid, kBuildThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_kmeans_d(const BuildArgs& a, int64_t nchunks, int B, cudaStream_t stream) {
  if (a.k <= 4) return launch_kmeans_t<T, D, 4>(a, nchunks, B, stream);
  if (a.k <= 8) return launch_kmeans_t<T, D, 8>(a, nchunks, B, stream);
  return launch_kmeans_t<T, D, 16>(a, nchunks, B, stream);
}

}  // namespace

// The new token's key and value rows of every (b, kvh) written into the cache
// at position seq_lens[b] - 1 (skipped when that is outside [0, Tmax)).
// One CTA per sequence; 16-byte copies.
__global__ void append_kv_kernel(uint4* K, uint4* V, int64_t sb, int64_t sh, int64_t st, const int64_t* seq_lens,
                                 const uint4* kn, const uint4* vn, int Hkv, int row16, int64_t Tmax) {
  // the next kernel (a decode launched as a programmatic dependent) may start
  // its input-free set-up now; it reads the cache only after this grid is done
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int n = Hkv * row16;
  // this thread's first piece of the new rows goes out before the sequence
  // length is known (the rows may sit in host memory: two round trips over
  // the host link would otherwise follow one another)
  const int i0 = threadIdx.x;
  uint4 k0 = make_uint4(0, 0, 0, 0), v0 = k0;
  if (i0 < n) {
    k0 = kn[(int64_t)b * n + i0];
    v0 = vn[(int64_t)b * n + i0];
  }
  const int64_t t = seq_lens[b] - 1;
  if (t < 0 || t >= Tmax) return;
  for (int i = i0; i < n; i += blockDim.x) {
    const int h = i / row16, c = i % row16;
    const int64_t dst = b * sb + h * sh + t * st + c;
    const int64_t src = (int64_t)b * n + i;
    K[dst] = i == i0 ? k0 : kn[src];
    V[dst] = i == i0 ? v0 : vn[src];
  }
}

cudaError_t launch_append(void* K, void* V, const int64_t* kv_strides_elems, int elem_bytes, int d,
                          const int64_t* seq_lens, const void* kn, const void* vn, int B, int Hkv, int64_t Tmax,
                          cudaStream_t stream) {
  const int64_t per16 = 16 / elem_bytes;  // elements per 16-byte piece
  const int row16 = d * elem_bytes / 16;
  append_kv_kernel<<<B, 128, 0, stream>>>(static_cast<uint4*>(K), static_cast<uint4*>(V), kv_strides_elems[0] / per16,
                                          kv_strides_elems[1] / per16, kv_strides_elems[2] / per16, seq_lens,
                                          static_cast<const uint4*>(kn), static_cast<const uint4*>(vn), Hkv, row16,
                                          Tmax);
  return cudaGetLastError();
}

cudaError_t launch_build(const BuildArgs& a, int dtype, int d, int64_t nchunks, int B,
                         cudaStream_t stream) {
  if (dtype == LOD_DTYPE_F32) {
    return d == 64 ? launch_kmeans_d<float, 64>(a, nchunks, B, stream)
                   : launch_kmeans_d<float, 128>(a, nchunks, B, stream);
  }
  return d == 64 ? launch_kmeans_d<__nv_bfloat16, 64>(a, nchunks, B, stream)
                 : launch_kmeans_d<__nv_bfloat16, 128>(a, nchunks, B, stream);
}

}  // namespace lod
