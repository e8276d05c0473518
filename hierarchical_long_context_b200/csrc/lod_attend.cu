// lod_attend.cu -- LoD decode and prefill attention ("Level of Detail
// Attention", How It Works, paragraphs 2-3).
//
// Two kernels per batch of query rows (bf16 caches with d = 128 take the
// tensor-core scan of lod_scan_tc.cu, which hands the refine kernel each
// split's best groups instead of every group's score):
//
//  scan    grid (unit, split).  A unit is one KV head of one sequence with its
//          NQ query rows (decode: the g query heads; prefill: g heads x NP
//          positions).  A split stages a slice of rows in shared memory with
//          TMA bulk copies -- either visible group summaries (mean key, mean
//          value, count) or exact window/sink tokens -- and computes
//            pass 1  the scores of all its rows against the NQ queries,
//            then    per query row the max logit (score + ln count), and the
//                    group scores go to the workspace's score array,
//            pass 2  the weighted sum of its values,
//          leaving a partial softmax state (max, sum, acc[d]) over ALL its rows.
//  refine  one CTA per query row, launched as a programmatic dependent of the
//          scan.  It merges the split states, picks the top `top_groups`
//          groups from the unit's score array (or from the splits' best
//          groups), removes those groups'
//          coarse terms (they are replaced by finer entries), scores each
//          opened group's page summaries, opens the top `top_pages` pages and
//          adds their tokens exactly (values staged by TMA), adds the other
//          pages as coarse entries (page mean logit + ln count, page mean
//          value), and writes out = acc / sum and the log-sum-exp.
//
// Removing the opened groups after the fact (instead of holding them out of
// the scan) is numerically safe: the entries that replace an opened group --
// its pages, or their tokens -- carry at least the group's own mass (by
// Jensen's inequality, n exp(q.mean k) <= sum exp(q.k): the coarse term never
// overstates a group),
// so the final normaliser is never smaller than what was subtracted and the
// cancellation error stays at the fp32 rounding level of the output.
#include <type_traits>

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

// N consecutive elements from shared memory as floats (one vector load).
template <typename T, int N>
__device__ __forceinline__ void lds_f(const T* p, float (&v)[N]) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (N == 4) {
      const float4 a = *reinterpret_cast<const float4*>(p);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
      static_assert(N == 2, "unsupported f32 vector width");
      const float2 a = *reinterpret_cast<const float2*>(p);
      v[0] = a.x; v[1] = a.y;
    }
  } else if constexpr (N == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(a.x << 16);
    v[1] = __uint_as_float(a.x & 0xffff0000u);
    v[2] = __uint_as_float(a.y << 16);
    v[3] = __uint_as_float(a.y & 0xffff0000u);
  } else {
    static_assert(N == 2, "unsupported bf16 vector width");
    const uint32_t a = *reinterpret_cast<const uint32_t*>(p);
    v[0] = __uint_as_float(a << 16);
    v[1] = __uint_as_float(a & 0xffff0000u);
  }
}

// Read-only global loads as volatile asm: they keep their place in program
// order (the compiler neither sinks them to their first use nor merges them),
// so that loads meant to overlap are in flight together.
__device__ __forceinline__ uint4 ldv_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ int ldv_s32(const int32_t* p) {
  int v;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ int ldv_s16(const int16_t* p) {
  short v;
  asm volatile("ld.global.nc.s16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
template <typename T, int N>
__device__ __forceinline__ void ldv_f(const T* p, float (&v)[N]) {
  if constexpr (N * sizeof(T) == 16) {
    const uint4 a = ldv_u4(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(w[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  } else if constexpr (N * sizeof(T) == 8) {
    uint32_t x, y;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(x), "=r"(y) : "l"(p));
    if constexpr (sizeof(T) == 4) {
      v[0] = __uint_as_float(x);
      v[1] = __uint_as_float(y);
    } else {
      v[0] = __uint_as_float(x << 16);
      v[1] = __uint_as_float(x & 0xffff0000u);
      v[2] = __uint_as_float(y << 16);
      v[3] = __uint_as_float(y & 0xffff0000u);
    }
  } else {
    static_assert(N * sizeof(T) == 4 && sizeof(T) == 2, "unsupported vector width");
    uint32_t x;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(x) : "l"(p));
    v[0] = __uint_as_float(x << 16);
    v[1] = __uint_as_float(x & 0xffff0000u);
  }
}

// The 4-bit codes of a lane's channels (nibbles 0..DPL-1 of w) as float
// pairs.  Nibble i is placed into the mantissa of 2^23 in place (2^23 +
// 2^(4i) code, exact) and one packed fma scales it back: x * 2^-4i -
// 2^(23-4i) = code, exactly.
template <int DPL>
__device__ __forceinline__ void lane_nibbles(uint32_t w, float2 (&c)[DPL / 2]) {
  c[0] = ffma2(make_float2(__uint_as_float(0x4B000000u | (w & 0xFu)), __uint_as_float(0x4B000000u | (w & 0xF0u))),
               make_float2(1.0f, 0.0625f), make_float2(-8388608.0f, -524288.0f));
  if constexpr (DPL == 4)
    c[1] = ffma2(make_float2(__uint_as_float(0x4B000000u | (w & 0xF00u)), __uint_as_float(0x4B000000u | (w & 0xF000u))),
                 make_float2(1.0f / 256.0f, 1.0f / 4096.0f), make_float2(-32768.0f, -2048.0f));
}

// Sum over the warp of 16 per-lane values: lane l receives the total of value
// l >> 1 (each step halves the values a lane keeps and exchanges the other half).
__device__ __forceinline__ float transpose_sum16(float (&v)[16], int lane) {
#pragma unroll
  for (int h = 8, b = 16; h >= 1; h >>= 1, b >>= 1) {
    const bool up = (lane & b) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float send = up ? v[j] : v[j + h];
      const float keep = up ? v[j + h] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, b);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// The 4-bit codes of `lane`'s DPL channels in one member-ordered row.
template <int D, int DPL>
__device__ __forceinline__ uint32_t lane_codes(const uint8_t* row, int lane) {
  if constexpr (DPL == 4) {
    return *reinterpret_cast<const uint16_t*>(row + lane * 2);
  } else {
    static_assert(DPL == 2, "channels per lane");
    return row[lane];
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

// An opened group (refine kernel).
struct Cand {
  float s;     // scale * q.mean_k
  int id;      // group id within the unit (chunk * k + slot), -1 = none
  int meta;    // the group's gMeta word
};

// ------------------------------------------------------------------ scan

constexpr int kSlab = 64;    // rows per pipeline stage
constexpr int kStages = 3;   // TMA ring depth

template <typename T, int D, int NQ>
struct ScanSmem {
  static constexpr size_t stage_bytes = (size_t)kSlab * D * sizeof(T);      // K or V of one slab
  static constexpr size_t off_K = 0;                                        // [kStages][kSlab][D]
  static constexpr size_t off_V = kStages * stage_bytes;                    // [kStages][kSlab][D]
  static constexpr size_t off_S = 2 * kStages * stage_bytes;                // float [NQ][kSlab]
  static constexpr size_t off_P = off_S + sizeof(float) * NQ * kSlab;       // float [kSlab][NQ]
  static constexpr size_t off_lnc = off_P + sizeof(float) * NQ * kSlab;     // float [kStages][kSlab]
  static constexpr size_t off_pos = off_lnc + sizeof(float) * kStages * kSlab;  // int64 [kStages][kSlab]
  static constexpr size_t off_corr = off_pos + sizeof(int64_t) * kStages * kSlab;  // float [16]
  static constexpr size_t off_bar = off_corr + sizeof(float) * 16;          // uint64 [kStages]
  static constexpr size_t bytes = off_bar + 8 * kStages;
  // the final cross-warp reduction reuses the K ring
  static_assert(sizeof(float) * kWarps * NQ * D <= kStages * stage_bytes, "reduction scratch");
};

// Row e of a unit's row list: e < G_vis -> group summary e; then the sinks;
// then the window [ws, t_max].  Returns the token position (-1 for a group).
__device__ __forceinline__ int64_t row_pos(int64_t e, int64_t G_vis, int64_t ns, int64_t ws) {
  if (e < G_vis) return -1;
  e -= G_vis;
  return e < ns ? e : ws + (e - ns);
}

template <typename T, int D, int NQ>
__global__ void __launch_bounds__(kThreads, 2) scan_kernel(AttendArgs a) {
  constexpr int EPL = 16 / sizeof(T);  // elements per lane per 16-byte load
  constexpr int LPR = D / EPL;         // lanes per row
  constexpr int RPI = 32 / LPR;        // rows per warp per step
  constexpr int ROWB = D * sizeof(T);
  constexpr int SHIFT = ilog2(LPR) - ilog2(NQ);
  using SM = ScanSmem<T, D, NQ>;
  static_assert(NQ <= LPR, "each query row's score must land on its own lanes");
  static_assert(kSlab % (kWarps * RPI) == 0, "a slab is a whole number of warp steps");

  const int64_t u = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int li = lane % LPR, sub = lane / LPR;
  pdl_wait();  // inputs are read only after the preceding kernel completed
  pdl_launch_dependents();
  const UnitInfo ui = unit_info(a, u);

  extern __shared__ __align__(128) unsigned char smem[];
  T* Kr = reinterpret_cast<T*>(smem + SM::off_K);
  T* Vr = reinterpret_cast<T*>(smem + SM::off_V);
  float* S_s = reinterpret_cast<float*>(smem + SM::off_S);
  float* P_s = reinterpret_cast<float*>(smem + SM::off_P);
  float* lnc_s = reinterpret_cast<float*>(smem + SM::off_lnc);
  int64_t* pos_s = reinterpret_cast<int64_t*>(smem + SM::off_pos);
  float* corr_s = reinterpret_cast<float*>(smem + SM::off_corr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::off_bar);
  float* red = reinterpret_cast<float*>(smem);  // [kWarps][NQ][D] at the end

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

  // ---- this split's slice of the unit's row list
  const int64_t unit_kv = (int64_t)ui.b * a.Hkv + ui.kvh;
  int64_t G_vis = 0, ns = 0, ws = 0, e0 = 0, e1 = 0;
  if (t_max >= 0) {
    const int64_t bt = t_max / kChunk;
    const int64_t nw = a.window / kChunk;
    const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;  // visible chunks [0, wb)
    ws = wb * kChunk;
    G_vis = wb * a.k;
    ns = 0;  // the sinks are exact tokens added by the refine kernel
    const int64_t total = G_vis + ns + (t_max - ws + 1);
    const int64_t per = (total + a.nsplit - 1) / a.nsplit;
    e0 = s * per < total ? s * per : total;
    e1 = e0 + per < total ? e0 + per : total;
  }
  const int nslab = (int)((e1 - e0 + kSlab - 1) / kSlab);
  const T* Kb = static_cast<const T*>(a.K) + ui.b * a.sb + ui.kvh * a.sh;
  const T* Vb = static_cast<const T*>(a.V) + ui.b * a.sb + ui.kvh * a.sh;
  const T* gK = static_cast<const T*>(a.gK) + unit_kv * a.Cmax * a.k * D;
  const T* gV = static_cast<const T*>(a.gV) + unit_kv * a.Cmax * a.k * D;
  const int32_t* gM = a.gMeta + unit_kv * a.Cmax * a.k;  // size | page range per group
  const int64_t gcap = a.Cmax * a.k;
  const bool contiguous = a.st == D;

  // producer: stage slab i (rows [e0 + 64 i, ...)) into ring slot i % kStages
  auto issue = [&](int i) {
    const int st = i % kStages;
    const int64_t r0 = e0 + (int64_t)i * kSlab;
    const int64_t r1 = r0 + kSlab < e1 ? r0 + kSlab : e1;
    const int n = (int)(r1 - r0);
    T* kd = Kr + (size_t)st * kSlab * D;
    T* vd = Vr + (size_t)st * kSlab * D;
    if (lane == 0) mbar_arrive_expect(&full[st], (uint32_t)n * 2u * ROWB);
    __syncwarp();
    // group summaries: one contiguous run
    const int64_t g1 = r1 < G_vis ? r1 : G_vis;
    if (r0 < g1 && lane == 0) {
      bulk_g2s(kd, gK + r0 * D, (uint32_t)(g1 - r0) * ROWB, &full[st]);
      bulk_g2s(vd, gV + r0 * D, (uint32_t)(g1 - r0) * ROWB, &full[st]);
    }
    // tokens (sinks, then the window): runs of consecutive positions
    const int64_t t0 = r0 > G_vis ? r0 : G_vis;
    if (t0 < r1) {
      if (contiguous) {
        if (lane == 0) {
          // at most two runs: sinks [.., ns) and window [ws, ..)
          int64_t e = t0;
          while (e < r1) {
            const int64_t p = row_pos(e, G_vis, ns, ws);
            int64_t run_end = e - G_vis < ns ? G_vis + ns : r1;
            if (run_end > r1) run_end = r1;
            const uint32_t bytes = (uint32_t)(run_end - e) * ROWB;
            bulk_g2s(kd + (e - r0) * D, Kb + p * D, bytes, &full[st]);
            bulk_g2s(vd + (e - r0) * D, Vb + p * D, bytes, &full[st]);
            e = run_end;
          }
        }
      } else {
        for (int64_t e = t0 + lane; e < r1; e += 32) {
          const int64_t p = row_pos(e, G_vis, ns, ws);
          bulk_g2s(kd + (e - r0) * D, Kb + p * a.st, ROWB, &full[st]);
          bulk_g2s(vd + (e - r0) * D, Vb + p * a.st, ROWB, &full[st]);
        }
      }
    }
  };
  // row metadata of slab i (log count, -inf = skip; token position, or
  // -2 - gMeta word for a group)
  auto meta = [&](int i, int r) {
    const int st = i % kStages;
    const int64_t e = e0 + (int64_t)i * kSlab + r;
    float lc = -INFINITY;
    int64_t p = -1;
    if (e < e1) {
      if (e < G_vis) {
        const int mt = gM[e];
        const int cnt = mt & 0xffff;
        if (cnt > 0 && cnt <= kChunk) lc = __logf((float)cnt);
        else if (cnt > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
        p = -2 - (int64_t)mt;
      } else {
        p = row_pos(e, G_vis, ns, ws);
        lc = 0.f;
      }
    }
    lnc_s[st * kSlab + r] = lc;
    pos_s[st * kSlab + r] = p;
  };

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0)
    for (int i = 0; i < kStages - 1 && i < nslab; ++i) issue(i);
  for (int i = 0; i < kStages - 1 && i < nslab; ++i)
    for (int r = tid; r < kSlab; r += kThreads) meta(i, r);

  // ---- the query rows (pre-scaled), this lane's EPL dims of each.  Row slot
  // j of this lane holds query row (j ^ perm): every reduce-scatter step then
  // keeps the low half of the live slots and sends the high half, with no
  // per-lane selects.
  const int perm = (li >> SHIFT) & (NQ - 1);
  float2 q2[NQ][EPL / 2];
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    float f[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) f[e] = 0.f;
    const int r = j ^ perm;
    bool okr = false;
#pragma unroll
    for (int x = 0; x < NQ; ++x)
      if (x == r) okr = ok[x];
    if (okr) {
      const int hq = ui.kvh * a.g + (r % a.g);
      const int64_t pi = a.seq_lens ? 0 : a.pos_lo + ui.blk * a.NP + r / a.g;
      const T* qp = static_cast<const T*>(a.q) + (((int64_t)ui.b * a.Hq + hq) * a.Tq + pi) * D;
      load_f<T, EPL>(qp + li * EPL, f);
    }
#pragma unroll
    for (int e = 0; e < EPL; e += 2) q2[j][e / 2] = make_float2(f[e] * a.scale, f[e + 1] * a.scale);
  }

  // running state: query row `warp` (warp < NQ) keeps (m, l)
  float m_run = -INFINITY, l_run = 0.f;
  // P.V accumulators: one value row per warp step, lane owns DPL = d/32 dims
  constexpr int DPL = D / 32;
  float2 acc[NQ][DPL / 2];
#pragma unroll
  for (int r = 0; r < NQ; ++r)
#pragma unroll
    for (int e = 0; e < DPL / 2; ++e) acc[r][e] = make_float2(0.f, 0.f);
  bool alive = true;  // false after a copy timed out

  for (int i = 0; i < nslab && alive; ++i) {
    const int st = i % kStages;
    const int64_t r0 = e0 + (int64_t)i * kSlab;
    const int n = (int)((e1 - r0) < kSlab ? (e1 - r0) : kSlab);
    const T* Ks = Kr + (size_t)st * kSlab * D;
    const T* Vs = Vr + (size_t)st * kSlab * D;
    if (!mbar_wait(&full[st], (uint32_t)(i / kStages) & 1u, a.status)) alive = false;
    // ---- scores of this slab
    if (alive) {
#pragma unroll
      for (int base = 0; base < kSlab; base += kWarps * RPI) {
        const int row = base + warp * RPI + sub;
        float k[EPL];
        if (row < n) {
          uint4 raw = *reinterpret_cast<const uint4*>(Ks + row * D + li * EPL);
          unpack16<T>(raw, k);
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e) k[e] = 0.f;
        }
        float part[NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
          float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < EPL; e += 2) s2 = ffma2(q2[j][e / 2], make_float2(k[e], k[e + 1]), s2);
          part[j] = s2.x + s2.y;
        }
#pragma unroll
        for (int step = 0; step < ilog2(LPR); ++step) {
          const int msk = LPR >> (step + 1);
          const int live = NQ >> step;
          if (live > 1) {
#pragma unroll
            for (int j = 0; j < NQ / 2; ++j)
              if (j < live / 2) part[j] += __shfl_xor_sync(0xffffffffu, part[j + live / 2], msk);
          } else {
            part[0] += __shfl_xor_sync(0xffffffffu, part[0], msk);
          }
        }
        if (row < n && (li & ((1 << SHIFT) - 1)) == 0) S_s[perm * kSlab + row] = part[0];
      }
    }
    if (!__syncthreads_and(alive)) {
      alive = false;
      break;
    }
    // the ring slot of slab i-1 is free now: stage slab i + kStages - 1
    if (i + kStages - 1 < nslab) {
      if (warp == 0) issue(i + kStages - 1);
      for (int r = tid; r < kSlab; r += kThreads) meta(i + kStages - 1, r);
    }
    // ---- per query row: running max, weights, running sum, group scores
    if (warp < NQ) {
      const int r = warp;
      float lg[kSlab / 32], sc[kSlab / 32];
      bool live[kSlab / 32];
      float smax = -INFINITY;
#pragma unroll
      for (int x = 0; x < kSlab / 32; ++x) {
        const int row = lane + 32 * x;
        const float lc = row < n ? lnc_s[st * kSlab + row] : -INFINITY;
        const int64_t p = pos_s[st * kSlab + row];
        live[x] = ok[r] && lc != -INFINITY && (p < 0 || p <= t_row[r]);
        sc[x] = S_s[r * kSlab + row];
        lg[x] = live[x] ? sc[x] + lc : -INFINITY;
        smax = fmaxf(smax, lg[x]);
      }
      smax = warp_max(smax);
      const float mn = fmaxf(m_run, smax);
      const float corr = (m_run == -INFINITY || mn == -INFINITY) ? (m_run == -INFINITY ? 0.f : 1.f)
                                                                  : __expf(m_run - mn);
      float psum = 0.f;
#pragma unroll
      for (int x = 0; x < kSlab / 32; ++x) {
        const float p = live[x] ? __expf(lg[x] - mn) : 0.f;
        P_s[(lane + 32 * x) * NQ + r] = p;
        psum += p;
      }
      psum = warp_sum(psum);
      l_run = l_run * corr + psum;
      m_run = mn;
      if (lane == 0) corr_s[r] = corr;
      // group scores (-inf: not in this query row's softmax)
      float2* gsr = a.gsc + (u * NQ + r) * gcap;
#pragma unroll
      for (int x = 0; x < kSlab / 32; ++x) {
        const int row = lane + 32 * x;
        const int64_t pr = pos_s[st * kSlab + row];
        if (row < n && pr < 0)
          gsr[r0 + row] = make_float2(live[x] ? sc[x] : -INFINITY, __int_as_float((int)(-2 - pr)));
      }
    }
    __syncthreads();
    // ---- acc[r] = acc[r] * corr[r] + P[:, r] . V   (warp w: rows w, w+8, ...)
    float cr[NQ];
#pragma unroll
    for (int r = 0; r < NQ; ++r) cr[r] = corr_s[r];
#pragma unroll
    for (int r = 0; r < NQ; ++r)
#pragma unroll
      for (int e = 0; e < DPL / 2; ++e) acc[r][e] = make_float2(acc[r][e].x * cr[r], acc[r][e].y * cr[r]);
#pragma unroll 2
    for (int row = warp; row < n; row += kWarps) {
      if (lnc_s[st * kSlab + row] == -INFINITY) continue;
      float v[DPL];
      if constexpr (sizeof(T) == 2 && DPL == 4) {
        const uint2 rw = *reinterpret_cast<const uint2*>(Vs + row * D + lane * DPL);
        v[0] = __uint_as_float(rw.x << 16);
        v[1] = __uint_as_float(rw.x & 0xffff0000u);
        v[2] = __uint_as_float(rw.y << 16);
        v[3] = __uint_as_float(rw.y & 0xffff0000u);
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) v[i] = Elem<T>::to_f(Vs[row * D + lane * DPL + i]);
      }
      float p[NQ];
      if constexpr (NQ % 4 == 0) {
#pragma unroll
        for (int r = 0; r < NQ; r += 4) {
          const float4 pp = *reinterpret_cast<const float4*>(P_s + row * NQ + r);
          p[r] = pp.x;
          p[r + 1] = pp.y;
          p[r + 2] = pp.z;
          p[r + 3] = pp.w;
        }
      } else {
#pragma unroll
        for (int r = 0; r < NQ; ++r) p[r] = P_s[row * NQ + r];
      }
#pragma unroll
      for (int r = 0; r < NQ; ++r)
#pragma unroll
        for (int e = 0; e < DPL; e += 2)
          acc[r][e / 2] = ffma2(make_float2(p[r], p[r]), make_float2(v[e], v[e + 1]), acc[r][e / 2]);
    }
  }
  // drain: no copy may still be in flight when the CTA exits
  if (!alive) {
    for (int i = 0; i < nslab && i < kStages; ++i) (void)mbar_wait(&full[i], 0, a.status);
  }

  // ---- reduce the warps' accumulators
  __syncthreads();  // the K ring becomes the reduction buffer
#pragma unroll
  for (int r = 0; r < NQ; ++r)
#pragma unroll
    for (int e = 0; e < DPL; e += 2)
      *reinterpret_cast<float2*>(red + (warp * NQ + r) * D + lane * DPL + e) = acc[r][e / 2];
  if (warp < NQ && lane == 0) {
    corr_s[warp] = alive ? m_run : -INFINITY;
  }
  float* lsh = P_s;  // l per query row
  if (warp < NQ && lane == 0) lsh[warp] = alive ? l_run : 0.f;
  __syncthreads();
  float* part = a.part + ((u * a.nsplit + s) * NQ) * (int64_t)(D + 2);
  for (int idx = tid; idx < NQ * (D + 2); idx += kThreads) {
    const int r = idx / (D + 2), c = idx % (D + 2);
    float v;
    if (c == 0) {
      v = corr_s[r];
    } else if (c == 1) {
      v = lsh[r];
    } else {
      v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[(w * NQ + r) * D + (c - 2)];
    }
    part[idx] = v;
  }
}

// ------------------------------------------------------------------ refine

template <typename T, int D>
struct RefineSmem {
  static constexpr int ROWB = D * sizeof(T);
  static constexpr int kRows = 48;  // per warp: 32 exact tokens + 16 coarse page means
  static constexpr size_t off_V = 0;                                     // [kWarps][kRows][D] T
  static constexpr size_t off_q = (size_t)kWarps * kRows * ROWB;        // float [D]
  static constexpr size_t off_g = off_q + sizeof(float) * D;            // float [D+4]
  // per-warp final states reuse the value buffers (used only after the group loop)
  static constexpr size_t off_w = off_V;                                // float [kWarps][D+4]
  static constexpr size_t off_d = off_V + sizeof(float) * kWarps * (D + 4);  // float [kWarps][D+4]
  static_assert(2 * sizeof(float) * kWarps * (D + 4) <= off_q, "final states fit the value buffers");
  static constexpr size_t off_sc = off_g + sizeof(float) * (D + 4);     // float [kWarps][64]
  static constexpr size_t off_pos = off_sc + sizeof(float) * kWarps * 64;     // int64 [kWarps][32]
  static constexpr size_t off_c = off_pos + sizeof(int64_t) * kWarps * 32;    // Cand [kMaxTopGroups]
  static constexpr size_t off_key = off_c + sizeof(Cand) * kMaxTopGroups + 16;  // uint64 [kWarps][32]
  static constexpr size_t off_wb = off_key + 8 * kWarps * 32;                  // uint64 [kWarps]
  static constexpr size_t off_bar = off_wb + 8 * kWarps + 16;
  static constexpr size_t bytes = off_bar + 8 * kWarps + 16;
  // group selection: the survivors of the bound reuse the value buffers
  static constexpr int kSurvCap = (int)(off_q / 8);
  static_assert(ROWB > 256 || bytes <= 113 * 1024, "two CTAs per SM for rows of up to 256 bytes");
};

// Scores of up to 32 d-rows against q, loaded with coalesced 16-byte loads:
// each half (or quarter) of the warp reads one whole row per step and the
// row's score is reduced over its lanes.  rowptr(i) gives row i (valid for
// i < n).  Writes score i to out[i].  EVICT_FIRST: rows read once (L2 policy).
template <typename T, int D, int STEPS, bool EVICT_FIRST = false, typename RowPtr>
__device__ __forceinline__ void rows_dot_coalesced(int n, RowPtr rowptr, const float (&qv)[16 / sizeof(T)],
                                                   float* out) {
  constexpr int EPL = 16 / sizeof(T);
  constexpr int LPR = D / EPL;
  constexpr int RPI = 32 / LPR;  // STEPS: loads in flight per lane per round
  const int lane = threadIdx.x & 31;
  const int li = lane % LPR, sub = lane / LPR;
  const uint64_t pol = EVICT_FIRST ? l2_policy_evict_first() : 0;
  for (int base = 0; base < n; base += STEPS * RPI) {
  uint4 raw[STEPS];
#pragma unroll
  for (int it = 0; it < STEPS; ++it) {
    const int i = base + it * RPI + sub;
    if (i < n) {
      const uint4* src = reinterpret_cast<const uint4*>(rowptr(i) + li * EPL);
      raw[it] = EVICT_FIRST ? ldg_hint(src, pol) : ldv_u4(src);
    }
  }
#pragma unroll
  for (int it = 0; it < STEPS; ++it) {
    if (base + it * RPI >= n) break;
    const int i = base + it * RPI + sub;
    float f[EPL];
    if (i < n) {
      unpack16<T>(raw[it], f);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) f[e] = 0.f;
    }
    float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) s2 = ffma2(make_float2(qv[e], qv[e + 1]), make_float2(f[e], f[e + 1]), s2);
    float sc = s2.x + s2.y;
#pragma unroll
    for (int msk = LPR / 2; msk > 0; msk >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, msk);
    if (li == 0 && i < n) out[i] = sc;
  }
  }
}

// Largest key over the CTA (every thread receives it); red: [kWarps] scratch.
__device__ __forceinline__ uint64_t block_max_key(uint64_t v, uint64_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t x = __shfl_xor_sync(0xffffffffu, v, o);
    v = x > v ? x : v;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  uint64_t r = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) r = red[w] > r ? red[w] : r;
  return r;
}

// Q4: three-tier INT4 (opened pages read from 4-bit codes; a.kv_bits == 4).
// SC: the groups come from the splits' best lists (a.cand, tensor-core scan)
// rather than from every group's score (a.gsc).
template <typename T, int D, int NQ, bool Q4, bool SC>
__global__ void __launch_bounds__(kThreads, 2) refine_kernel(AttendArgs a) {
  constexpr int DPL = D / 32;
  constexpr int EPL = 16 / sizeof(T);
  constexpr int LPR = D / EPL;
  constexpr int ROWB = D * sizeof(T);
  using SM = RefineSmem<T, D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  float* qs = reinterpret_cast<float*>(smem + SM::off_q);
  float* gstate = reinterpret_cast<float*>(smem + SM::off_g);
  float* wstate = reinterpret_cast<float*>(smem + SM::off_w);
  float* dstate = reinterpret_cast<float*>(smem + SM::off_d);
  float* sc_s = reinterpret_cast<float*>(smem + SM::off_sc);
  int64_t* posm_s = reinterpret_cast<int64_t*>(smem + SM::off_pos);
  Cand* win = reinterpret_cast<Cand*>(smem + SM::off_c);
  int* nwin_s = reinterpret_cast<int*>(smem + SM::off_c + sizeof(Cand) * kMaxTopGroups);
  uint64_t* keys_s = reinterpret_cast<uint64_t*>(smem + SM::off_key);
  uint64_t* wb_s = reinterpret_cast<uint64_t*>(smem + SM::off_wb);
  uint64_t* surv = reinterpret_cast<uint64_t*>(smem + SM::off_V);
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
  pdl_wait();  // the scan's partial states and group scores are visible from here on
  pdl_launch_dependents();
  // the sink tokens [0, min(sinks, window start)) are exact entries (last
  // warp); their rows go to L2 now, while the groups are selected
  const int64_t wsq = (t / kChunk - a.window / kChunk + 1) > 0 ? (t / kChunk - a.window / kChunk + 1) * kChunk : 0;
  const int64_t nsk = a.sinks < wsq ? a.sinks : wsq;
  const T* Kb = static_cast<const T*>(a.K) + b * a.sb + kvh * a.sh;
  const T* Vb = static_cast<const T*>(a.V) + b * a.sb + kvh * a.sh;
  if (warp == kWarps - 1)
    for (int64_t e = lane; e < nsk; e += 32)
      for (int o = 0; o < ROWB; o += 128) {
        prefetch_l2(reinterpret_cast<const char*>(Kb + e * a.st) + o);
        prefetch_l2(reinterpret_cast<const char*>(Vb + e * a.st) + o);
      }

  const int nsplit = a.nsplit;
  // the split states this thread merges (component c = tid of each), loaded
  // now so that the loads overlap the group selection
  constexpr int kPre = 8;
  const float* ps = a.part + (u * nsplit * NQ + r) * (int64_t)(D + 2);
  const int64_t pstride = (int64_t)NQ * (D + 2);
  float pre_m[kPre], pre_v[kPre];
#pragma unroll
  for (int sp = 0; sp < kPre; ++sp) {
    pre_m[sp] = -INFINITY;
    pre_v[sp] = 0.f;
    if (sp < nsplit && tid < D + 2) {
      pre_m[sp] = ps[sp * pstride];
      pre_v[sp] = ps[sp * pstride + tid];
    }
  }
  // ---- the top-G groups of this row (higher score first, then smaller id)
  if constexpr (SC) {
    // from the splits' own best G: every candidate's exact rank among them
    const SplitCand* cr = a.cand + (u * nsplit * NQ + r) * (int64_t)a.G;
    const int nall = nsplit * a.G;
    int* cmeta = reinterpret_cast<int*>(surv + nall);
    if (tid == 0) *nwin_s = 0;
    for (int x = tid; x < nall; x += kThreads) {
      const SplitCand c = cr[(int64_t)(x / a.G) * NQ * a.G + x % a.G];
      surv[x] = c.id >= 0 ? group_key(c.s, c.id) : 0ull;
      cmeta[x] = c.meta;
    }
    __syncthreads();
    for (int x = tid; x < nall; x += kThreads) {
      const uint64_t kx = surv[x];
      if (kx == 0ull) continue;
      int rx = 0;
      for (int y = 0; y < nall; ++y) rx += surv[y] > kx ? 1 : 0;
      if (rx < a.G) {
        win[rx].s = key_score(kx);
        win[rx].id = key_id(kx);
        win[rx].meta = cmeta[x];
        atomicMax(nwin_s, rx + 1);
      }
    }
  } else {
  // From the unit's score array: a bound that G distinct groups reach (the
  // G-th largest of a warp's per-thread best scores; the largest such bound
  // over the warps), the groups scoring at or above it (a few dozen), then
  // their exact ranks by (score, id).
    const int64_t wbq = t / kChunk - a.window / kChunk + 1;
    const int Gq = wbq > 0 ? (int)(wbq * a.k) : 0;  // visible groups of this row
    const float2* srow = a.gsc + (u * NQ + r) * (a.Cmax * a.k);
    constexpr int kSel = 8;  // scores per thread kept in registers (up to 2048 groups)
    const bool in_regs = Gq <= kSel * kThreads;
    const int ns = (Gq + kThreads - 1) / kThreads;  // register slots in use (uniform)
    float sv[kSel];
    float bs = -INFINITY;
    int bi = 0x7fffffff;
    if (in_regs) {
#pragma unroll
      for (int e = 0; e < kSel; ++e) {
        const int i = tid + e * kThreads;
        sv[e] = -INFINITY;
        if (e < ns && i < Gq) sv[e] = srow[i].x;
      }
#pragma unroll
      for (int e = 0; e < kSel; ++e)
        if (e < ns && sv[e] > bs) {  // first occurrence: the smaller id wins a tie
          bs = sv[e];
          bi = tid + e * kThreads;
        }
    } else {
      for (int i = tid; i < Gq; i += kThreads) {
        const float si = srow[i].x;
        if (si > bs) {
          bs = si;
          bi = i;
        }
      }
    }
    // the warp's G-th largest per-thread best (32-bit orderable score; equal
    // scores counted with their multiplicity): G distinct groups reach it
    const uint32_t tb32 = okey32(bs);
    uint32_t kk = tb32, wbound = 0;
    int cum = 0;
    for (int it = 0; it < a.G; ++it) {
      const uint32_t mx = __reduce_max_sync(0xffffffffu, kk);
      if (mx == 0u) break;
      const unsigned eq = __ballot_sync(0xffffffffu, kk == mx);
      cum += __popc(eq);
      if (kk == mx) kk = 0u;
      if (cum >= a.G) {
        wbound = mx;
        break;
      }
    }
    uint32_t* wb32 = reinterpret_cast<uint32_t*>(wb_s);
    int* wtot = reinterpret_cast<int*>(keys_s);
    if (lane == 0) wb32[warp] = wbound;
    __syncthreads();
    uint32_t lo = 1u;  // groups with a score at or above the bound survive
#pragma unroll
    for (int w = 0; w < kWarps; ++w) lo = max(lo, wb32[w]);
    // survivors: per-slot ballots give each warp its count and each lane its offset
    const uint32_t lt = (1u << lane) - 1u;
    int n = 0;
    if (in_regs) {
      uint32_t msk[kSel];
      int wcount = 0;
#pragma unroll
      for (int e = 0; e < kSel; ++e) {
        msk[e] = e < ns ? __ballot_sync(0xffffffffu, okey32(sv[e]) >= lo) : 0u;
        wcount += __popc(msk[e]);
      }
      if (lane == 0) wtot[warp] = wcount;
      __syncthreads();
      int base = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int c = wtot[w];
        base += w < warp ? c : 0;
        n += c;
      }
#pragma unroll
      for (int e = 0; e < kSel; ++e) {
        if (e >= ns) break;
        if ((msk[e] >> lane) & 1u) {
          const int pos = base + __popc(msk[e] & lt);
          if (pos < SM::kSurvCap) surv[pos] = group_key(sv[e], tid + e * kThreads);
        }
        base += __popc(msk[e]);
      }
    } else {
      if (tid == 0) wtot[kWarps] = 0;
      __syncthreads();
      for (int i = tid; i < Gq; i += kThreads) {
        const float si = srow[i].x;
        if (okey32(si) >= lo) {
          const int pos = atomicAdd(&wtot[kWarps], 1);
          if (pos < SM::kSurvCap) surv[pos] = group_key(si, i);
        }
      }
    }
    __syncthreads();
    if (!in_regs) n = wtot[kWarps];
    const int nwin = n < a.G ? n : a.G;
    if (n <= 64) {  // four threads rank each survivor
      const int x = tid >> 2, qq = tid & 3;
      const uint64_t kx = x < n ? surv[x] : 0ull;
      int rx = 0;
      for (int y = qq; y < n; y += 4) rx += surv[y] > kx ? 1 : 0;
      rx += __shfl_xor_sync(0xffffffffu, rx, 1);
      rx += __shfl_xor_sync(0xffffffffu, rx, 2);
      if (x < n && qq == 0 && rx < nwin) {
        win[rx].s = key_score(kx);
        win[rx].id = key_id(kx);
      }
    } else if (n <= SM::kSurvCap) {
      for (int x = tid; x < n; x += kThreads) {
        const uint64_t kx = surv[x];
        int rx = 0, y = 0;
        for (; y + 1 < n; y += 2) {
          const ulonglong2 pq = *reinterpret_cast<const ulonglong2*>(surv + y);
          rx += (pq.x > kx ? 1 : 0) + (pq.y > kx ? 1 : 0);
        }
        if (y < n) rx += surv[y] > kx ? 1 : 0;
        if (rx < nwin) {
          win[rx].s = key_score(kx);
          win[rx].id = key_id(kx);
        }
      }
    } else {  // more survivors than the buffer holds: one rank at a time
      uint64_t last = ~0ull;
      for (int x = 0; x < nwin; ++x) {
        uint64_t bk = 0;
        for (int i = tid; i < Gq; i += kThreads) {
          const uint64_t kv = group_key(srow[i].x, i);
          if (kv < last && kv > bk) bk = kv;
        }
        bk = block_max_key(bk, wb_s);
        if (tid == 0) {
          win[x].s = key_score(bk);
          win[x].id = key_id(bk);
        }
        last = bk;
      }
    }
    if (tid == 0) *nwin_s = nwin;
  }
  if (tid < D + 2) {
    // ---- merge the split states (thread c owns component c: m, l, acc[])
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < kPre; ++sp) M = fmaxf(M, pre_m[sp]);
    for (int sp = kPre; sp < nsplit; ++sp) M = fmaxf(M, ps[sp * pstride]);
    float v = 0.f;
    if (tid == 0) {
      v = M;
    } else {
#pragma unroll
      for (int sp = 0; sp < kPre; ++sp)
        if (pre_m[sp] != -INFINITY) v = fmaf(pre_v[sp], __expf(pre_m[sp] - M), v);
      for (int sp = kPre; sp < nsplit; ++sp) {
        const float ms = ps[sp * pstride];
        if (ms != -INFINITY) v = fmaf(ps[sp * pstride + tid], __expf(ms - M), v);
      }
    }
    gstate[tid] = v;
  }
  __syncthreads();
  const int nwin = *nwin_s;
  const float M = gstate[0];

  // this lane's slice of q in the coalesced layout (dims (lane % LPR) * EPL ..)
  float qv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) qv[e] = qs[(lane % LPR) * EPL + e];

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
  const T* mK = static_cast<const T*>(a.mK) + unit_kv * a.Cmax * kChunk * D;
  const T* mV = static_cast<const T*>(a.mV) + unit_kv * a.Cmax * kChunk * D;
  T* myV = Vst + warp * SM::kRows * D;
  float* mysc = sc_s + warp * 64;
  const T** mykp = reinterpret_cast<const T**>(posm_s) + warp * 32;
  uint32_t phase = 0;
  // member key rows scored per round of coalesced loads; rows past the first
  // round are brought into L2 while that round is in flight
  constexpr int kMemberSteps = 8;
  constexpr int kFirstRound = kMemberSteps * (32 / LPR);
  const uint64_t l2once = l2_policy_evict_first();  // member rows are read once
  // One batch of up to 32 exact tokens (lane e: `ev`, key and value rows
  // `krow`, `vrow`) and up to 32 coarse entries (lane p: `cvb`, logit `lgc`,
  // value row `crow`): the value rows are staged in shared memory by TMA
  // while the key rows are scored with coalesced loads, then everything
  // enters the warp's online softmax state.
  auto batch = [&](bool ev, const T* krow, const T* vrow, bool cvb, float lgc, const T* crow) {
    const unsigned vm = __ballot_sync(0xffffffffu, ev);
    const unsigned cmb = __ballot_sync(0xffffffffu, cvb);
    if (!(vm | cmb)) return;
    // exact tokens are packed: the valid ones take ranks 0..nvalid-1 in lane
    // order, for their key pointers, scores, weights and staged value rows
    const int nvalid = __popc(vm);
    const int my_rank = __popc(vm & ((1u << lane) - 1u));
    if (lane == 0) mbar_arrive_expect(&bar[warp], (uint32_t)(nvalid + __popc(cmb)) * ROWB);
    __syncwarp();
    if (ev) bulk_g2s_hint(myV + my_rank * D, vrow, ROWB, &bar[warp], l2once);
    if (cvb) bulk_g2s(myV + (32 + lane) * D, crow, ROWB, &bar[warp]);
    if (ev) {
      mykp[my_rank] = krow;
      if (my_rank >= kFirstRound)
        for (int o = 0; o < ROWB; o += 128) prefetch_l2(reinterpret_cast<const char*>(krow) + o);
    }
    __syncwarp();
    rows_dot_coalesced<T, D, kMemberSteps, true>(nvalid, [&](int i) { return mykp[i]; }, qv, mysc + 32);
    __syncwarp();
    const float lge = ev ? mysc[32 + my_rank] : -INFINITY;
    const float lgcb = cvb ? lgc : -INFINITY;
    const float bm = warp_max(fmaxf(lge, lgcb));
    const float mn = fmaxf(m, bm);
    const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
    const float pe = ev ? __expf(lge - mn) : 0.f;
    const float pc = cvb ? __expf(lgcb - mn) : 0.f;
    l = l * corr + warp_sum(pe + pc);
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] *= corr;
    m = mn;
    if (ev) mysc[my_rank] = pe;  // the exact tokens' weights in rank order
    const bool okw = mbar_wait(&bar[warp], phase, a.status);
    phase ^= 1u;
    if (!okw) {
      (void)mbar_wait(&bar[warp], phase ^ 1u, a.status);  // drain before the buffer is reused
      __syncwarp();
      return;
    }
    __syncwarp();
    // exact tokens: the packed rows in rank order, four per step
    int j = 0;
    for (; j + 4 <= nvalid; j += 4) {
      const float4 p4 = *reinterpret_cast<const float4*>(mysc + j);
      float v0[DPL], v1[DPL], v2[DPL], v3[DPL];
      lds_f<T, DPL>(myV + (j + 0) * D + lane * DPL, v0);
      lds_f<T, DPL>(myV + (j + 1) * D + lane * DPL, v1);
      lds_f<T, DPL>(myV + (j + 2) * D + lane * DPL, v2);
      lds_f<T, DPL>(myV + (j + 3) * D + lane * DPL, v3);
#pragma unroll
      for (int i = 0; i < DPL; i += 2) {
        float2 a2 = make_float2(acc[i], acc[i + 1]);
        a2 = ffma2(make_float2(p4.x, p4.x), make_float2(v0[i], v0[i + 1]), a2);
        a2 = ffma2(make_float2(p4.y, p4.y), make_float2(v1[i], v1[i + 1]), a2);
        a2 = ffma2(make_float2(p4.z, p4.z), make_float2(v2[i], v2[i + 1]), a2);
        a2 = ffma2(make_float2(p4.w, p4.w), make_float2(v3[i], v3[i + 1]), a2);
        acc[i] = a2.x;
        acc[i + 1] = a2.y;
      }
    }
    for (; j < nvalid; ++j) {
      const float pj = mysc[j];
      float v[DPL];
      lds_f<T, DPL>(myV + j * D + lane * DPL, v);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, v[i], acc[i]);
    }
    // coarse entries, in lane order
    unsigned rest = cmb;
    while (rest) {
      const int jc = __ffs((int)rest) - 1;
      rest &= rest - 1;
      const float pj = __shfl_sync(0xffffffffu, pc, jc);
      float v[DPL];
      lds_f<T, DPL>(myV + (32 + jc) * D + lane * DPL, v);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, v[i], acc[i]);
    }
    __syncwarp();
  };
  // Three-tier INT4 ("Level of Detail Attention", the paragraph after the
  // quality tables: only the selected pages are decompressed): up to two
  // opened pages (rows ra/rb of the member-ordered codes, na/nb members, page
  // slots sa/sb, all relative to the unit) per batch, with the coarse entries
  // of `batch`.  The pages' codes and (scale, low) quantisers are staged by
  // TMA; a member's logit is q.low + sum_j (q_j scale_j) code_j and the values
  // enter as scale_j sum_r p_r code_rj + low_j sum_r p_r per page.  Lane e is
  // member e % 16 of page e / 16.
  auto batch_q = [&](int npg, int64_t ra, int na, int64_t sa, int64_t rb, int nb, int64_t sb, bool cvb, float lgc,
                     const T* crow) {
    const unsigned cmb = __ballot_sync(0xffffffffu, cvb);
    if (npg == 0 && !cmb) return;
    unsigned char* stg = reinterpret_cast<unsigned char*>(myV);
    constexpr int PB = 8 * D;  // one staged piece: 16 rows of d/2 codes, or d (scale, low) pairs
    const uint8_t* qKu = a.qK + unit_kv * a.Cmax * kChunk * (D / 2);
    const uint8_t* qVu = a.qV + unit_kv * a.Cmax * kChunk * (D / 2);
    const float2* qKsu = a.qKs + unit_kv * a.Cmax * a.P * D;
    const float2* qVsu = a.qVs + unit_kv * a.Cmax * a.P * D;
    if (lane == 0) {
      uint32_t bytes = (uint32_t)__popc(cmb) * ROWB;
      if (npg > 0) bytes += (uint32_t)(na * D + 2 * PB);
      if (npg > 1) bytes += (uint32_t)(nb * D + 2 * PB);
      mbar_arrive_expect(&bar[warp], bytes);
      if (npg > 0) {
        bulk_g2s_hint(stg + 0 * PB, qKu + ra * (D / 2), (uint32_t)(na * (D / 2)), &bar[warp], l2once);
        bulk_g2s_hint(stg + 2 * PB, qVu + ra * (D / 2), (uint32_t)(na * (D / 2)), &bar[warp], l2once);
        bulk_g2s(stg + 4 * PB, qKsu + sa * D, PB, &bar[warp]);
        bulk_g2s(stg + 6 * PB, qVsu + sa * D, PB, &bar[warp]);
      }
      if (npg > 1) {
        bulk_g2s_hint(stg + 1 * PB, qKu + rb * (D / 2), (uint32_t)(nb * (D / 2)), &bar[warp], l2once);
        bulk_g2s_hint(stg + 3 * PB, qVu + rb * (D / 2), (uint32_t)(nb * (D / 2)), &bar[warp], l2once);
        bulk_g2s(stg + 5 * PB, qKsu + sb * D, PB, &bar[warp]);
        bulk_g2s(stg + 7 * PB, qVsu + sb * D, PB, &bar[warp]);
      }
    }
    __syncwarp();
    if (cvb) bulk_g2s(myV + (32 + lane) * D, crow, ROWB, &bar[warp]);
    float qd[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) qd[i] = qs[lane * DPL + i];
    const bool okw = mbar_wait(&bar[warp], phase, a.status);
    phase ^= 1u;
    if (!okw) {
      (void)mbar_wait(&bar[warp], phase ^ 1u, a.status);  // drain before the buffer is reused
      __syncwarp();
      return;
    }
    // logits of the pair's members
    float lge = -INFINITY;
    bool ev = false;
#pragma unroll 1
    for (int x = 0; x < npg; ++x) {
      const int n = x == 0 ? na : nb;
      const float2* kq = reinterpret_cast<const float2*>(stg + (4 + x) * PB);
      const uint8_t* kc = stg + x * PB;
      float2 qsc[DPL / 2];
      float qlo = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; i += 2) {
        const float2 z0 = kq[lane * DPL + i], z1 = kq[lane * DPL + i + 1];
        qsc[i / 2] = make_float2(qd[i] * z0.x, qd[i + 1] * z1.x);
        qlo = fmaf(qd[i], z0.y, qlo);
        qlo = fmaf(qd[i + 1], z1.y, qlo);
      }
      qlo = warp_sum(qlo);
      float part[kPage];
#pragma unroll
      for (int r = 0; r < kPage; ++r) {
        part[r] = 0.f;
        if (r < n) {
          float2 cw[DPL / 2];
          lane_nibbles<DPL>(lane_codes<D, DPL>(kc + r * (D / 2), lane), cw);
          float2 sd = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < DPL / 2; ++i) sd = ffma2(qsc[i], cw[i], sd);
          part[r] = sd.x + sd.y;
        }
      }
      const float tot = transpose_sum16(part, lane) + qlo;  // member lane >> 1
      const float v = __shfl_sync(0xffffffffu, tot, (2 * (lane & 15)) & 31);
      if ((lane >> 4) == x && (lane & 15) < n) {
        lge = v;
        ev = true;
      }
    }
    const float lgcb = cvb ? lgc : -INFINITY;
    const float bm = warp_max(fmaxf(lge, lgcb));
    const float mn = fmaxf(m, bm);
    const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
    const float pe = ev ? __expf(lge - mn) : 0.f;
    const float pc = cvb ? __expf(lgcb - mn) : 0.f;
    l = l * corr + warp_sum(pe + pc);
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] *= corr;
    m = mn;
    mysc[lane] = pe;  // member r of page x at 16 x + r
    __syncwarp();
#pragma unroll 1
    for (int x = 0; x < npg; ++x) {
      const int n = x == 0 ? na : nb;
      const float2* vq = reinterpret_cast<const float2*>(stg + (6 + x) * PB);
      const uint8_t* vc = stg + (2 + x) * PB;
      float2 ac[DPL / 2];
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) ac[i] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int r = 0; r < kPage; ++r) {
        if (r < n) {
          const float pr = mysc[16 * x + r];
          float2 cw[DPL / 2];
          lane_nibbles<DPL>(lane_codes<D, DPL>(vc + r * (D / 2), lane), cw);
#pragma unroll
          for (int i = 0; i < DPL / 2; ++i) ac[i] = ffma2(make_float2(pr, pr), cw[i], ac[i]);
          ps += pr;
        }
      }
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const float2 z = vq[lane * DPL + i];
        const float a_i = (i & 1) ? ac[i / 2].y : ac[i / 2].x;
        acc[i] = fmaf(z.x, a_i, fmaf(z.y, ps, acc[i]));
      }
    }
    // coarse entries, in lane order
    unsigned rest = cmb;
    while (rest) {
      const int jc = __ffs((int)rest) - 1;
      rest &= rest - 1;
      const float pj = __shfl_sync(0xffffffffu, pc, jc);
      float v[DPL];
      lds_f<T, DPL>(myV + (32 + jc) * D + lane * DPL, v);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, v[i], acc[i]);
    }
    __syncwarp();
  };
  // the sink tokens (last warp)
  if (warp == kWarps - 1) {
    for (int64_t e0 = 0; e0 < nsk; e0 += 32)
      batch(e0 + lane < nsk, Kb + (e0 + lane) * a.st, Vb + (e0 + lane) * a.st, false, 0.f, pV);
  }
  for (int w = warp; w < nwin; w += kWarps) {
    const float gs = win[w].s;
    const int gid = win[w].id;
    const int64_t c = gid / a.k;
    // size and page range: the gMeta word the scan stored beside the score
    int meta;
    if constexpr (SC)
      meta = win[w].meta;
    else
      meta = __float_as_int(a.gsc[(u * NQ + r) * (a.Cmax * a.k) + gid].y);
    const int gcnt = meta & 0xffff;
    const int p0 = (meta >> 16) & 0xff, p1 = (meta >> 24) & 0xff;
    // one round trip: the group's mean value, its pages' member counts and
    // offsets (lane l: page p0 + l) and their summary scores (volatile loads
    // keep this order; the counts are first needed after the page choice)
    const bool prange_ok = !(p1 < p0 || p1 > a.P || p1 - p0 > 32);
    const int np = prange_ok ? p1 - p0 : 0;
    float gv[DPL];
    ldv_f<T, DPL>(gV + (int64_t)gid * D + lane * DPL, gv);
    int cntp = 0, begp = 0;
    if (lane < np) {
      cntp = ldv_s32(pC + c * a.P + p0 + lane);
      begp = ldv_s16(pB + c * a.P + p0 + lane);
    }
    const T* pKc = pK + (c * a.P + (prange_ok ? p0 : 0)) * D;
    // (two-tier LoD opens the group whole: no page scores)
    rows_dot_coalesced<T, D, 8>(a.TP > 0 ? np : 0, [&](int i) { return pKc + (int64_t)i * D; }, qv, mysc);
    int open_slot[kMaxTopPages];
#pragma unroll
    for (int x = 0; x < kMaxTopPages; ++x) open_slot[x] = -1;
    // remove this group's coarse term: exp(s + ln n - M) * (1, gV)
    if (gcnt > 0 && gcnt <= kChunk) {
      const float e = __expf(gs + __logf((float)gcnt) - M);
      dl -= e;
#pragma unroll
      for (int i = 0; i < DPL; ++i) dacc[i] = fmaf(-e, gv[i], dacc[i]);
    } else {
      if (lane == 0) set_status(a.status, LOD_ST_BAD_COUNT);
    }
    if (!prange_ok) {
      if (lane == 0) set_status(a.status, LOD_ST_BAD_PAGE);
    } else {
      // the page summary scores
      __syncwarp();
      const float sc = lane < np ? mysc[lane] : -INFINITY;
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
      // coarse entries: the unopened pages of this group (lane p), staged with the first batch
      // (two-tier LoD has no page tier: no coarse pages)
      const bool cv = a.TP > 0 && lane < np && !is_open && cntp > 0 && cntp <= kPage;
      if (a.TP > 0 && lane < np && !is_open && (cntp <= 0 || cntp > kPage)) set_status(a.status, LOD_ST_BAD_COUNT);
      const unsigned cm = __ballot_sync(0xffffffffu, cv);
      const float lgc = cv ? sc + __logf((float)cntp) : -INFINITY;
      // exact members, 32 per batch.  Paged: lane e -> (opened page e/16,
      // member e%16).  Two-tier LoD (top_pages = 0): the whole group, one
      // contiguous run of the member-ordered copies from its first page.
      const int b0 = __shfl_sync(0xffffffffu, begp, 0);
      const bool whole = a.TP == 0;
      const bool okrun = gcnt > 0 && gcnt <= kChunk && b0 >= 0 && b0 + gcnt <= kChunk;
      if (whole && !okrun && lane == 0) set_status(a.status, LOD_ST_BAD_MEMBER);
      const int nbatch = whole ? (okrun ? (gcnt + 31) / 32 : 0) : (nopen * kPage + 31) / 32;
      if constexpr (Q4) {  // three-tier INT4: the opened pages two per batch
        const int npair = (nopen + 1) / 2;
        for (int bt = 0; bt < (npair > 0 ? npair : 1); ++bt) {
          int sa = -1, sb = -1;
#pragma unroll
          for (int y = 0; y < kMaxTopPages; ++y) {
            if (y == 2 * bt) sa = open_slot[y];
            if (y == 2 * bt + 1) sb = open_slot[y];
          }
          int na = __shfl_sync(0xffffffffu, cntp, (sa - p0) & 31);
          int ba = __shfl_sync(0xffffffffu, begp, (sa - p0) & 31);
          int nb = __shfl_sync(0xffffffffu, cntp, (sb - p0) & 31);
          int bb = __shfl_sync(0xffffffffu, begp, (sb - p0) & 31);
          if (sa < 0) na = 0;
          if (sb < 0) nb = 0;
          if (na > kPage || nb > kPage) {
            if (lane == 0) set_status(a.status, LOD_ST_BAD_PAGE);
            if (na > kPage) na = 0;
            if (nb > kPage) nb = 0;
          }
          if ((na > 0 && (ba < 0 || ba + na > kChunk)) || (nb > 0 && (bb < 0 || bb + nb > kChunk))) {
            if (lane == 0) set_status(a.status, LOD_ST_BAD_MEMBER);
            if (na > 0 && (ba < 0 || ba + na > kChunk)) na = 0;
            if (nb > 0 && (bb < 0 || bb + nb > kChunk)) nb = 0;
          }
          if (na <= 0) {  // pack a lone page into the first place
            na = nb;
            ba = bb;
            sa = sb;
            nb = 0;
          }
          const int npg = (na > 0 ? 1 : 0) + (nb > 0 ? 1 : 0);
          batch_q(npg, c * kChunk + ba, na, c * a.P + sa, c * kChunk + bb, nb, c * a.P + sb, bt == 0 && cv, lgc,
                  pV + (c * a.P + p0 + lane) * D);
        }
      } else
      for (int bt = 0; bt < (nbatch > 0 ? nbatch : 1); ++bt) {
        const int e = bt * 32 + lane;
        const int x = e / kPage, mi = e % kPage;
        int slot = -1;
#pragma unroll
        for (int y = 0; y < kMaxTopPages; ++y)
          if (y == x) slot = open_slot[y];
        const int sl_lane = slot >= 0 ? slot - p0 : 0;
        int n_of = __shfl_sync(0xffffffffu, cntp, sl_lane & 31);
        int b_of = __shfl_sync(0xffffffffu, begp, sl_lane & 31);
        bool ev = x < nopen && slot >= 0 && mi < n_of;
        if (whole) {
          ev = okrun && e < gcnt;
          n_of = 1;
          b_of = b0 + e;
        }
        if (ev && !whole && n_of > kPage) {
          set_status(a.status, LOD_ST_BAD_PAGE);
          ev = false;
        }
        if (ev && !whole && (b_of < 0 || b_of + n_of > kChunk)) {
          set_status(a.status, LOD_ST_BAD_MEMBER);
          ev = false;
        }
        if (whole) {
          n_of = 0;
        }
        // the page's members are consecutive rows of the member-ordered copies
        const int64_t row = c * kChunk + (ev ? b_of + (whole ? 0 : mi) : 0);
        batch(ev, mK + row * D, mV + row * D, bt == 0 && cv, lgc, pV + (c * a.P + p0 + lane) * D);
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
  // (the value staging buffers are free now and hold the per-warp states)
  __syncthreads();
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

template <typename T, int D, int NQ>
cudaError_t launch_t(const AttendArgs& a, const TcMaps* maps, cudaStream_t stream) {
  const int nsplit = a.nsplit;
  const int64_t npos = a.seq_lens ? 1 : a.pos_hi - a.pos_lo;
  const int64_t rows = (int64_t)a.B * a.Hq * npos;
  cudaError_t e = cudaSuccess;
  if (a.units > 0 && nsplit > 0) {
    if (maps) {
      e = launch_scan_tc(a, *maps, NQ, stream);
    } else if constexpr (NQ <= 8) {
      auto sk = scan_kernel<T, D, NQ>;
      const size_t smem = ScanSmem<T, D, NQ>::bytes;
      e = set_smem_once<scan_kernel<T, D, NQ>>(smem);
      if (e != cudaSuccess) return e;
      e = launch_pdl(sk, dim3((unsigned)a.units, (unsigned)nsplit), dim3(kThreads), smem, stream, a);
    } else {
      return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  if (rows > 0) {
    const bool q4 = a.kv_bits == 4;
    const size_t smem = RefineSmem<T, D>::bytes;
    void (*rk)(AttendArgs) = nullptr;
    if (a.cand) {  // tensor-core scan: bf16, d = 128
      if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
        rk = q4 ? refine_kernel<T, D, NQ, true, true> : refine_kernel<T, D, NQ, false, true>;
        e = q4 ? set_smem_once<refine_kernel<T, D, NQ, true, true>>(smem)
               : set_smem_once<refine_kernel<T, D, NQ, false, true>>(smem);
      } else {
        return cudaErrorInvalidValue;
      }
    } else {
      rk = q4 ? refine_kernel<T, D, NQ, true, false> : refine_kernel<T, D, NQ, false, false>;
      e = q4 ? set_smem_once<refine_kernel<T, D, NQ, true, false>>(smem)
             : set_smem_once<refine_kernel<T, D, NQ, false, false>>(smem);
    }
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

template <typename T, int D>
cudaError_t launch_nq(const AttendArgs& a, int NQ, const TcMaps* maps, cudaStream_t stream) {
  switch (NQ) {
    case 1: return launch_t<T, D, 1>(a, maps, stream);
    case 2: return launch_t<T, D, 2>(a, maps, stream);
    case 4: return launch_t<T, D, 4>(a, maps, stream);
    case 8: return launch_t<T, D, 8>(a, maps, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace


cudaError_t launch_attend(const AttendArgs& a, int dtype, int d, int NQ, const TcMaps* maps,
                          cudaStream_t stream) {
  if (dtype == LOD_DTYPE_F32)
    return d == 64 ? launch_nq<float, 64>(a, NQ, nullptr, stream) : launch_nq<float, 128>(a, NQ, nullptr, stream);
  return d == 64 ? launch_nq<__nv_bfloat16, 64>(a, NQ, nullptr, stream)
                 : launch_nq<__nv_bfloat16, 128>(a, NQ, maps, stream);
}

}  // namespace lod
