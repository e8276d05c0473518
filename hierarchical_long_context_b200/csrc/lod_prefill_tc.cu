// lod_prefill_tc.cu -- grouped chunked prefill of LoD attention on tcgen05
// tensor cores (bf16 caches, d = 128).
//
// What each query row computes is "Level of Detail Attention", How It Works
// paragraphs 2-3 (the same as lod_decode).  How the rows are organised
// follows "Coarse Semantic Blocks for Efficient Training-Free Sparse
// Attention", Abstract: in prefill, the queries that pick the same block are
// handled together, which keeps prefill fast.  Here the block is an index
// group, and the rows that opened it share one dense tensor-core tile.  Per
// wave of query chunks:
//
//  A  pf_scan_kernel   one CTA per 128 query rows of one KV head (128/g
//                      positions x g heads, all in one query chunk, so they
//                      share one visible index).  S = Q K^T on the tensor
//                      cores against every visible group summary, the sinks
//                      and the causal block window (keys on N), one online
//                      softmax per row (group logits carry + ln count), and
//                      O += P V on the tensor cores; each row's top-G groups
//                      are kept in its thread's registers.  The epilogue
//                      removes the top-G groups' coarse terms (finer entries
//                      replace them in B), stores the row state, and counts
//                      the (row, group) pairs of every group.
//  plan, scatter       counting sort of the pairs by (KV head, group) and
//                      the work items (one group's pairs, up to kItemRows).
//  B  pf_pair_kernel   per work item the group's member keys and values and
//                      its page summaries are staged once.  For tiles of 128
//                      pairs (the rows that opened the group) S = Q K_g^T
//                      and Sp = Q pK^T score every member and page summary;
//                      each row opens its top_pages pages, and O = P [V_g; pV]
//                      adds the opened members exactly and the unopened pages
//                      as coarse entries (page mean value, logit + ln count)
//                      in one MMA chain.  The pair's normalised partial
//                      (log-sum-exp, bf16 output) is stored.
//  merge               per row: the row state and its pairs' partials in one
//                      softmax; out and lse.
//
// Softmax arithmetic is in log2 units (logit * log2 e) with ex2 on the SFU.
// Removing the opened groups' coarse terms after the fact is numerically
// safe for the reason given in lod_attend.cu: the entries that replace a
// group carry at least its mass (n exp(q.mean k) <= sum exp(q.k)).
#include <cudaTypedefs.h>

#include "lod_internal.cuh"
#include "lod_tc.cuh"

namespace lod {

namespace {

constexpr int D = 128;
constexpr int kRows = 128;                      // query rows (or pairs) per tile: MMA M
constexpr uint32_t kTileBytes = 128 * D * 2;    // one 128 x 128 bf16 operand tile
constexpr uint32_t kHalf = kTileBytes / 2;      // one 64-column half of it
constexpr float kTau2 = 12.f;                   // weights reach at most 2^kTau2 before the reference max moves
constexpr int kStateStride = 132;               // floats per row state: m, l, -, -, acc[128]

__device__ __forceinline__ uint32_t sw_off(int row, int chunk16) {  // 16-byte chunk of a 128B-swizzled row
  return (uint32_t)(row * 128 + (((chunk16 & 7) ^ (row & 7)) << 4));
}

// ================================================================== phase A

constexpr int kThreadsA = 192;   // warp 0 TMA, warp 1 MMA issue, warps 2-5 softmax
constexpr int kBarSoftA = 1;

struct SmemA {
  static constexpr size_t off_Q = 0;                          // [2 halves][128][128 B]
  static constexpr size_t off_K = off_Q + kTileBytes;         // [2 stages]
  static constexpr size_t off_V = off_K + 2 * kTileBytes;     // [2 stages]
  static constexpr size_t off_P = off_V + 2 * kTileBytes;     // [2 halves][128][128 B]
  static constexpr size_t off_meta = off_P + kTileBytes;      // int [2][128]
  static constexpr size_t off_lnc = off_meta + 2 * 128 * 4;   // float [2][128]
  static constexpr size_t off_stash = off_lnc + 2 * 128 * 4;  // float [128][33]
  static constexpr int kBars = 15;
  static constexpr size_t off_bar = off_stash + 128 * 33 * 4;
  static constexpr size_t off_misc = off_bar + 8 * kBars;     // tmem slot, abort flag
  static constexpr size_t bytes = off_misc + 16 + 1024;
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Insert (v, id) into the descending list (s, ix) of GM entries: every entry
// from the first one v beats moves down by one place.  Ties keep the earlier
// entry first (ids arrive in increasing order, so the lower id wins).
template <int GM>
__device__ __forceinline__ void topk_insert(float (&s)[GM], int (&ix)[GM], float v, int id) {
  bool act = false;
  float cs = v;
  int ci = id;
#pragma unroll
  for (int k = 0; k < GM; ++k) {
    act = act || (v > s[k]);
    const float ts = s[k];
    const int ti = ix[k];
    if (act) {
      s[k] = cs;
      ix[k] = ci;
      cs = ts;
      ci = ti;
    }
  }
}

template <int GM>
__device__ __forceinline__ float topk_kth(const float (&s)[GM], int G) {
  float t = s[GM - 1];
#pragma unroll
  for (int k = 0; k < GM; ++k)
    if (k == G - 1) t = s[k];
  return t;
}

template <int GM>
__global__ void __launch_bounds__(kThreadsA, 1)
    pf_scan_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ PrefillArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  unsigned char* Qs = sm + SmemA::off_Q;
  unsigned char* Kring = sm + SmemA::off_K;
  unsigned char* Vring = sm + SmemA::off_V;
  unsigned char* Ps = sm + SmemA::off_P;
  int* meta_s = reinterpret_cast<int*>(sm + SmemA::off_meta);
  float* lnc_s = reinterpret_cast<float*>(sm + SmemA::off_lnc);
  float* stash = reinterpret_cast<float*>(sm + SmemA::off_stash);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(sm + SmemA::off_bar);
  uint64_t* kempty = kfull + 2;
  uint64_t* vfull = kempty + 2;
  uint64_t* vempty = vfull + 2;
  uint64_t* s_full = vempty + 2;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* fin = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SmemA::off_misc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + SmemA::off_misc + 4);

  // ---- the tile: heaviest (latest positions) first
  const int RP = kRows / a.g;                                // positions per tile
  const int64_t npos = a.w_hi - a.w_lo;
  const int64_t nblk = (npos + RP - 1) / RP;
  const int64_t units = (int64_t)a.B * a.Hkv;
  const int64_t blk = nblk - 1 - (int64_t)blockIdx.x / units;
  const int64_t u = (int64_t)blockIdx.x % units;             // b * Hkv + kvh
  const int b = (int)(u / a.Hkv), kvh = (int)(u % a.Hkv);
  const int64_t pos0 = a.w_lo + blk * RP;                    // first q position of the tile
  const int64_t pos_end = (pos0 + RP < a.w_hi) ? pos0 + RP : a.w_hi;
  const int64_t t0 = a.q_begin + pos0, t_max = a.q_begin + pos_end - 1;
  const int64_t bt = t0 / kChunk;                            // the tile's query chunk
  const int64_t nw = a.window / kChunk;
  const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
  const int64_t ws = wb * kChunk;                            // window start
  const int64_t G_vis = wb * a.k;
  const int64_t nsk = a.sinks < ws ? a.sinks : ws;
  const int gt = (int)((G_vis + 127) / 128);
  const int st_ = (int)((nsk + 127) / 128);
  const int ntile = gt + st_ + (int)((t_max - ws + 1 + 127) / 128);
  const int64_t Gcap = a.Cmax * a.k;
  const int64_t grow0 = u * Gcap;                            // this unit's first group row

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&vfull[i], 1 + 32);
      mbar_init(&vempty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_s = 0;
    fence_mbar_init();
    tc::prefetch_tensormap(&maps.gK);
    tc::prefetch_tensormap(&maps.gV);
    tc::prefetch_tensormap(&maps.K);
    tc::prefetch_tensormap(&maps.V);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
  // ---- the query tile (softmax warps): row r = position r / g, head r % g
  if (warp >= 2) {
    const int r = tid - 64;  // 0..127: each thread stages one row
    const int64_t pi = pos0 + r / a.g;
    const int hq = kvh * a.g + r % a.g;
    const bool okr = pi < pos_end;
    const __nv_bfloat16* src = a.q + (((int64_t)b * a.Hq + hq) * a.Tq + (okr ? pi : 0)) * D;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 v = okr ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(Qs + (c >> 3) * kHalf + sw_off(r, c)) = v;
    }
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_s) return false;
    if (mbar_wait(bar, parity, a.status)) return true;
    *abort_s = 1;
    return false;
  };
  const uint64_t l2pol = l2_policy_evict_first();

  if (warp == 0) {
    // ================================================================ producer
    const int32_t* gM = a.gMeta + grow0;
    int kissued = 0, vissued = 0;
    for (int i = 0; i < ntile; ++i) {
      const int st = i & 1;
      unsigned char* kd = Kring + st * kTileBytes;
      unsigned char* vd = Vring + st * kTileBytes;
      const bool grp = i < gt, snk = !grp && i < gt + st_;
      const int pos = grp ? 0 : (snk ? (i - gt) * 128 : (int)(ws + (int64_t)(i - gt - st_) * 128));
      const int row = grp ? (int)(grow0 + (int64_t)i * 128) : 0;
      if (i >= 2 && !wait(&kempty[st], ((i - 2) >> 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect(&kfull[st], kTileBytes);
        if (grp) {
          tc::tma_load_2d(kd, &maps.gK, 0, row, &kfull[st], l2pol);
          tc::tma_load_2d(kd + kHalf, &maps.gK, 64, row, &kfull[st], l2pol);
        } else {
          tc::tma_load_4d(kd, &maps.K, 0, pos, kvh, b, &kfull[st], l2pol);
          tc::tma_load_4d(kd + kHalf, &maps.K, 64, pos, kvh, b, &kfull[st], l2pol);
        }
      }
      ++kissued;
      if (i >= 2 && !wait(&vempty[st], ((i - 2) >> 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect(&vfull[st], kTileBytes);
        if (grp) {
          tc::tma_load_2d(vd, &maps.gV, 0, row, &vfull[st], l2pol);
          tc::tma_load_2d(vd + kHalf, &maps.gV, 64, row, &vfull[st], l2pol);
        } else {
          tc::tma_load_4d(vd, &maps.V, 0, pos, kvh, b, &vfull[st], l2pol);
          tc::tma_load_4d(vd + kHalf, &maps.V, 64, pos, kvh, b, &vfull[st], l2pol);
        }
      }
      if (grp) {  // the groups' size and page range (zero past the visible ones)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int r = lane + 32 * k4;
          const int64_t gid = (int64_t)i * 128 + r;
          const bool v = gid < G_vis;
          cp_async4_zfill(meta_s + st * 128 + r, v ? gM + gid : gM, v);
        }
      }
      cp_async_mbar_arrive_noinc(&vfull[st]);
      ++vissued;
    }
    cp_async_wait_all();
    if (*abort_s && lane == 0) {  // copies still in flight land before the CTA ends
      for (int i = kissued - 1; i >= 0 && i >= kissued - 2; --i)
        (void)mbar_wait(&kfull[i & 1], (uint32_t)(i >> 1) & 1u, a.status);
      for (int i = vissued - 1; i >= 0 && i >= vissued - 2; --i)
        (void)mbar_wait(&vfull[i & 1], (uint32_t)(i >> 1) & 1u, a.status);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issue
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      const uint32_t idO = tc::idesc_bf16(128, 128, false, true);
      const uint32_t qb = smem_u32(Qs), pb = smem_u32(Ps);
      auto mma2 = [&](int j) -> bool {  // O += P_j V_j
        if (!wait(p_full, (uint32_t)j & 1u)) return false;
        if (!wait(&vfull[j & 1], (uint32_t)(j >> 1) & 1u)) return false;
        tc::fence_after_sync();
        const uint32_t vb = smem_u32(Vring + (j & 1) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = tc::desc_kmajor_sw128(pb + (kk >> 2) * kHalf + (kk & 3) * 32);
          const uint64_t bd = tc::desc_mnmajor_sw128(vb + kk * 2048, kHalf);
          tc::mma_bf16(tmem + 256, ad, bd, idO, j > 0 || kk > 0);
        }
        tc::mma_commit(&vempty[j & 1]);
        tc::mma_commit(o_done);
        return true;
      };
      bool go = true, any = false;
      for (int i = 0; i < ntile && go; ++i) {
        if (!wait(&kfull[i & 1], (uint32_t)(i >> 1) & 1u)) break;
        if (i >= 2 && !wait(&s_free[i & 1], (uint32_t)((i - 2) >> 1) & 1u)) break;
        tc::fence_after_sync();
        const uint32_t kb = smem_u32(Kring + (i & 1) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = tc::desc_kmajor_sw128(qb + (kk >> 2) * kHalf + (kk & 3) * 32);
          const uint64_t bd = tc::desc_kmajor_sw128(kb + (kk >> 2) * kHalf + (kk & 3) * 32);
          tc::mma_bf16(tmem + (uint32_t)(i & 1) * 128, ad, bd, idS, kk > 0);
        }
        tc::mma_commit(&kempty[i & 1]);
        tc::mma_commit(&s_full[i & 1]);
        any = true;
        if (i >= 1) go = mma2(i - 1);
        if (go && i == ntile - 1) go = mma2(i);
      }
      if (any) {
        tc::mma_commit(fin);
        (void)mbar_wait(fin, 0, a.status);
      }
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // query row of this thread (and key row it stages)
    const uint32_t tl = (uint32_t)(32 * q4) << 16;
    const int64_t pi = pos0 + r / a.g;
    const int hq = kvh * a.g + r % a.g;
    const bool valid = pi < pos_end;
    const int64_t t_row = a.q_begin + pi;
    const float scl = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    float ts[GM];
    int ti[GM];
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      ts[k] = -INFINITY;
      ti[k] = -1;
    }
    float thr = -INFINITY;
    float* my_stash = stash + r * 33;
    bool alive = true;
    for (int i = 0; i < ntile; ++i) {
      const int st = i & 1;
      const bool grp = i < gt, snk = !grp && i < gt + st_;
      const int64_t kpos0 = grp ? 0 : (snk ? (int64_t)(i - gt) * 128 : ws + (int64_t)(i - gt - st_) * 128);
      // (a failed wait in a group tile is carried to that tile's softmax
      // barrier, where the four warps leave the loop together)
      alive = __all_sync(0xffffffffu, wait(&s_full[st], (uint32_t)(i >> 1) & 1u) &&
                                          wait(&vfull[st], (uint32_t)(i >> 1) & 1u));
      if (!alive && !grp) break;
      float s[128];
      if (alive) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tc::tmem_ld32(tmem + tl + (uint32_t)st * 128 + 32 * c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) s[32 * c + e] = v[e];
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[st]);
      }
      // key row r of this tile: its bias (group tiles) and whether it is in
      // no row's softmax (its value row is then zeroed: MMA 2 must not meet
      // NaN or Inf from rows that are not inputs of this call)
      bool dead = false;
      if (!alive) {
      } else if (grp) {
        const int mt = meta_s[st * 128 + r];
        const int c = mt & 0xffff;
        const int64_t gid = (int64_t)i * 128 + r;
        const bool okg = gid < G_vis && c > 0 && c <= kChunk;
        if (gid < G_vis && c > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
        lnc_s[st * 128 + r] = okg ? log2f((float)c) : -INFINITY;
        dead = !okg;
      } else {
        const int64_t kp = kpos0 + r;
        dead = snk ? kp >= nsk : kp > t_max;
      }
      if (dead) {
        unsigned char* vd = Vring + st * kTileBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(vd + h * kHalf + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      float xm = -INFINITY;
      if (grp) {
        // every group's ln count is in lnc_s past this barrier
        if (bar_red_or(kBarSoftA, 128, !alive)) {
          alive = false;
          break;
        }
        const float* lc = lnc_s + st * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float lv[32];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lc + 32 * c + 4 * e4);
            lv[4 * e4] = l4.x;
            lv[4 * e4 + 1] = l4.y;
            lv[4 * e4 + 2] = l4.z;
            lv[4 * e4 + 3] = l4.w;
          }
          // the raw scores of the groups in this row's softmax (-inf otherwise)
          float cm = -INFINITY;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            s[32 * c + e] = (valid && lv[e] != -INFINITY) ? s[32 * c + e] : -INFINITY;
            cm = fmaxf(cm, s[32 * c + e]);
          }
          // top-G: only a chunk holding a score above the current G-th best
          // is scanned (rare once the first tiles have filled the list)
          const bool cand = cm > thr;
          if (__any_sync(0xffffffffu, cand)) {
            if (cand) {
#pragma unroll
              for (int e = 0; e < 32; ++e) my_stash[e] = s[32 * c + e];
              for (int e = 0; e < 32; ++e) {
                const float v = my_stash[e];
                if (v > thr) {
                  topk_insert<GM>(ts, ti, v, (int)((int64_t)i * 128 + 32 * c + e));
                  thr = topk_kth<GM>(ts, a.G);
                }
              }
            }
            __syncwarp();
          }
          // the logits in log2 units: score * scale * log2 e + log2 count
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            s[32 * c + e] = fmaf(s[32 * c + e], scl, lv[e]);
            xm = fmaxf(xm, s[32 * c + e]);
          }
        }
      } else {
        const int64_t lim = snk ? nsk - 1 : t_row;  // keys at positions kpos0 + j <= lim
        const int64_t rel = valid ? lim - kpos0 : -1;
        if (rel >= 127) {
#pragma unroll
          for (int j = 0; j < 128; ++j) {
            s[j] *= scl;
            xm = fmaxf(xm, s[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 128; ++j) {
            s[j] = j <= rel ? s[j] * scl : -INFINITY;
            xm = fmaxf(xm, s[j]);
          }
        }
      }
      // the reference max moves when a logit exceeds it by more than kTau2
      const bool need = xm > m + kTau2;
      bool waited = false;
      if (__any_sync(0xffffffffu, need)) {
        const float mn = need ? xm : m;
        const float corr = (m == -INFINITY) ? 0.f : ex2_approx(m - mn);
        l *= corr;
        m = mn;
        if (i > 0) {
          alive = __all_sync(0xffffffffu, wait(o_done, (uint32_t)(i - 1) & 1u));
          waited = true;
          if (alive) {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float ov[32];
              tc::tmem_ld32(tmem + tl + 256 + 32 * c, ov);
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] *= corr;
              tc::tmem_st32(tmem + tl + 256 + 32 * c, ov);
            }
          }
        }
      }
      // the weights into P (free once MMA 2 of the previous tile is done)
      if (i > 0 && !waited) alive = __all_sync(0xffffffffu, wait(o_done, (uint32_t)(i - 1) & 1u)) && alive;
      if (!alive) break;
      const float mu = m == -INFINITY ? 0.f : m;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = ex2_approx(s[8 * c + e] - mu);
          l += p[e];
        }
        const uint4 w = make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                                   pack_bf16x2(p[6], p[7]));
        *reinterpret_cast<uint4*>(Ps + (c >> 3) * kHalf + sw_off(r, c)) = w;
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---------------------------------------------------------------- epilogue
    if (alive && ntile > 0) alive = __all_sync(0xffffffffu, wait(o_done, (uint32_t)(ntile - 1) & 1u));
    tc::fence_after_sync();
    const int64_t wr = ((int64_t)b * a.Hq + hq) * a.NW + (pi - a.w_lo);  // wave row
    const int64_t orow = ((int64_t)b * a.Hq + hq) * a.Tq + pi;
    float w[GM], lcnt[GM];
    int nsel = 0;
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      w[k] = 0.f;
      lcnt[k] = 0.f;
      if (k < a.G && ti[k] >= 0) {
        const int c = a.gMeta[grow0 + ti[k]] & 0xffff;
        lcnt[k] = log2f((float)(c > 0 ? c : 1));
        ++nsel;
      }
    }
    const float mu = m == -INFINITY ? 0.f : m;
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      if (k < nsel) {
        w[k] = ex2_approx(fmaf(ts[k], scl, lcnt[k]) - mu);
        l -= w[k];
      }
    }
    float* stp = a.state + wr * kStateStride;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float ov[32];
      tc::tmem_ld32(tmem + tl + 256 + 32 * c, ov);
      if (valid && alive) {
#pragma unroll
        for (int k = 0; k < GM; ++k) {
          if (k < nsel) {
            const uint4* gv = reinterpret_cast<const uint4*>(a.gV + (grow0 + ti[k]) * D + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 raw = __ldg(gv + q);
              const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                ov[8 * q + 2 * e] = fmaf(-w[k], __uint_as_float(wd[e] << 16), ov[8 * q + 2 * e]);
                ov[8 * q + 2 * e + 1] = fmaf(-w[k], __uint_as_float(wd[e] & 0xffff0000u), ov[8 * q + 2 * e + 1]);
              }
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(stp + 4 + 32 * c + 4 * q) =
              make_float4(ov[4 * q], ov[4 * q + 1], ov[4 * q + 2], ov[4 * q + 3]);
      }
    }
    if (valid) {
      if (alive) {
        stp[0] = m;
        stp[1] = l;
      } else {
        stp[0] = -INFINITY;
        stp[1] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < GM; ++k) {
        if (k < a.G) {
          const int gid = (alive && k < nsel) ? ti[k] : -1;
          a.sel[wr * a.G + k] = gid;
          if (a.sel_groups) a.sel_groups[orow * a.G + k] = gid;
          a.pos[wr * a.G + k] = gid >= 0 ? atomicAdd(a.cnt + grow0 + gid, 1) : -1;
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ================================================================== plan, scatter

constexpr int kPlanThreads = 1024;

// Exclusive prefix sums of the per-group pair counts (off) and the work
// items: group gflat with c pairs gives ceil(c / item_rows) items
// {gflat, first pair, pairs}.
__global__ void __launch_bounds__(kPlanThreads) pf_plan_kernel(const __grid_constant__ PrefillArgs a) {
  __shared__ int wsum[2][32];
  __shared__ long long carry[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int64_t base = 0; base < a.Gtot; base += kPlanThreads) {
    const int64_t gf = base + tid;
    const int c = gf < a.Gtot ? a.cnt[gf] : 0;
    const int ni = (c + a.item_rows - 1) / a.item_rows;
    int xp = c, xi = ni;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yp = __shfl_up_sync(0xffffffffu, xp, o), yi = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) {
        xp += yp;
        xi += yi;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = xp;
      wsum[1][warp] = xi;
    }
    __syncthreads();
    if (warp == 0) {
      int sp = wsum[0][lane], si = wsum[1][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yp = __shfl_up_sync(0xffffffffu, sp, o), yi = __shfl_up_sync(0xffffffffu, si, o);
        if (lane >= o) {
          sp += yp;
          si += yi;
        }
      }
      wsum[0][lane] = sp;
      wsum[1][lane] = si;
    }
    __syncthreads();
    const long long bp = carry[0] + (warp > 0 ? wsum[0][warp - 1] : 0) + xp - c;
    const long long bi = carry[1] + (warp > 0 ? wsum[1][warp - 1] : 0) + xi - ni;
    if (gf < a.Gtot) {
      a.off[gf] = (int32_t)bp;
      for (int x = 0; x < ni; ++x) {
        const int n = c - x * a.item_rows < a.item_rows ? c - x * a.item_rows : a.item_rows;
        a.items[bi + x] = make_int4((int)gf, (int)(bp + (long long)x * a.item_rows), n, 0);
      }
    }
    __syncthreads();
    if (tid == 0) {
      carry[0] += wsum[0][31];
      carry[1] += wsum[1][31];
    }
    __syncthreads();
  }
  if (tid == 0) *a.n_items = (int32_t)carry[1];
}

// Every (row, group) pair into its group's run of the pair list.
__global__ void __launch_bounds__(256) pf_scatter_kernel(const __grid_constant__ PrefillArgs a) {
  const int64_t n = (int64_t)a.B * a.Hq * a.NW * a.G;
  for (int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * 256) {
    const int64_t wr = idx / a.G;
    const int64_t pr = wr % a.NW;
    if (a.w_lo + pr >= a.w_hi) continue;
    const int gid = a.sel[idx];
    if (gid < 0) continue;
    const int64_t bh = wr / a.NW;
    const int64_t u = (bh / a.Hq) * a.Hkv + (bh % a.Hq) / a.g;
    a.list[a.off[u * a.Cmax * a.k + gid] + a.pos[idx]] = (int32_t)idx;
  }
}

// ================================================================== phase B

constexpr int kThreadsB = 160;   // warp 0 TMA + MMA issue, warps 1-4 one pair per thread
constexpr int kBarSoftB = 2;
constexpr size_t kSmemBData = 216 * 1024;  // operand regions (laid out per work item)

struct SmemB {
  static constexpr size_t off_misc = kSmemBData;           // per-item info, page counts, barriers
  static constexpr size_t off_lpc = off_misc + 64;         // float [16] log2 page counts
  static constexpr size_t off_bar = off_lpc + 64;
  static constexpr int kBars = 6;
  static constexpr size_t off_tmem = off_bar + 8 * kBars;
  static constexpr size_t bytes = off_tmem + 16 + 1024;
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

struct ItemInfo {
  int n, np, p0, ok;
  int start, count, R, shared_qp;
  int64_t c, u;
  uint32_t off_kg, off_vg, off_q, off_p;
};

__global__ void __launch_bounds__(kThreadsB, 1)
    pf_pair_kernel(const __grid_constant__ PairMaps maps, const __grid_constant__ PrefillArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  ItemInfo* info = reinterpret_cast<ItemInfo*>(sm + SmemB::off_misc);
  float* lpc_s = reinterpret_cast<float*>(sm + SmemB::off_lpc);
  uint64_t* gfull = reinterpret_cast<uint64_t*>(sm + SmemB::off_bar);
  uint64_t* q_full = gfull + 1;
  uint64_t* s_full = q_full + 1;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_done = p_full + 1;
  uint64_t* o_free = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SmemB::off_tmem);
  unsigned char* PKs = sm;             // [2 halves][16 rows][128 B]
  unsigned char* PVs = sm + 4096;

  if (tid == 0) {
    mbar_init(gfull, 1);
    mbar_init(q_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(o_free, 4);
    fence_mbar_init();
    tc::prefetch_tensormap(&maps.mK);
    tc::prefetch_tensormap(&maps.mV);
    tc::prefetch_tensormap(&maps.pK);
    tc::prefetch_tensormap(&maps.pV);
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n_items = *a.n_items;
  const int64_t Gcap = a.Cmax * a.k;
  const float scl = a.scale_log2;
  const int G = a.G, TP = a.TP;
  uint32_t T = 0;      // tiles processed by this CTA (barrier phases)
  uint32_t ngrp = 0;   // items with a staged group (gfull phases)
  bool alive = true;

  for (int it = blockIdx.x; it < n_items && alive; it += gridDim.x) {
    // ---- the item: its group, bounds-checked, and the operand layout
    if (tid == 0) {
      const int4 item = a.items[it];
      const int64_t gflat = item.x;
      const int64_t u = gflat / Gcap, gid = gflat % Gcap, c = gid / a.k;
      const int meta = a.gMeta[gflat];
      const int n = meta & 0xffff, p0 = (meta >> 16) & 0xff, p1 = (meta >> 24) & 0xff;
      const int64_t pslot = (u * a.Cmax + c) * a.P;
      bool ok = n >= 1 && n <= kChunk && p0 < p1 && p1 <= a.P && p1 - p0 == (n + kPage - 1) / kPage;
      if (!ok) set_status(a.status, n > kChunk ? LOD_ST_BAD_COUNT : LOD_ST_BAD_PAGE);
      const int off = ok ? (int)a.pBeg[pslot + p0] : 0;
      if (ok && (off < 0 || off + n > kChunk)) {
        set_status(a.status, LOD_ST_BAD_MEMBER);
        ok = false;
      }
      ItemInfo f;
      f.n = ok ? n : 16;
      f.np = ok ? p1 - p0 : 1;
      f.p0 = p0;
      f.ok = ok;
      f.start = item.y;
      f.count = item.z;
      f.c = c;
      f.u = u;
      f.R = ok ? (n + 31) / 32 * 32 : 32;
      const uint32_t kg = (uint32_t)f.R * 256;  // one operand: 2 halves x R rows x 128 B
      const int n16 = (f.n + 15) / 16 * 16;
      const uint32_t pbytes = (uint32_t)((n16 + 16 + 63) / 64) * kHalf;
      f.off_kg = 8192;
      f.off_vg = 8192 + kg;
      f.off_q = 8192 + 2 * kg;
      f.shared_qp = f.off_q + kTileBytes + pbytes > kSmemBData;
      f.off_p = f.shared_qp ? f.off_q : f.off_q + kTileBytes;
      *info = f;
      if (ok) {
        mbar_arrive_expect(gfull, 2 * kg + 2 * 4096);
        const int row0 = (int)((u * a.Cmax + c) * kChunk + off);
        for (int bx = 0; bx < f.R / 32; ++bx)
          for (int h = 0; h < 2; ++h) {
            tc::tma_load_2d(sm + f.off_kg + h * (f.R * 128) + bx * 4096, &maps.mK, 64 * h, row0 + 32 * bx, gfull,
                            0x1000000000000000ull);
            tc::tma_load_2d(sm + f.off_vg + h * (f.R * 128) + bx * 4096, &maps.mV, 64 * h, row0 + 32 * bx, gfull,
                            0x1000000000000000ull);
          }
        for (int h = 0; h < 2; ++h) {
          tc::tma_load_2d(PKs + h * 2048, &maps.pK, 64 * h, (int)(pslot + p0), gfull, 0x1000000000000000ull);
          tc::tma_load_2d(PVs + h * 2048, &maps.pV, 64 * h, (int)(pslot + p0), gfull, 0x1000000000000000ull);
        }
      } else {
        mbar_arrive(gfull);
      }
    }
    __syncthreads();
    const ItemInfo f = *info;
    const int n16 = (f.n + 15) / 16 * 16;
    const int ntiles = (f.count + kRows - 1) / kRows;
    unsigned char* KG = sm + f.off_kg;
    unsigned char* VG = sm + f.off_vg;
    unsigned char* Qs = sm + f.off_q;
    unsigned char* Ps = sm + f.off_p;

    if (warp == 0) {
      // ============================================================ MMA issue
      if (lane == 0) {
        bool go = mbar_wait(gfull, ngrp & 1u, a.status);
        const uint32_t idS = tc::idesc_bf16(128, n16, false, false);
        const uint32_t idP = tc::idesc_bf16(128, 16, false, false);
        const uint32_t idO = tc::idesc_bf16(128, 128, false, true);
        const uint32_t qb = smem_u32(Qs), kb = smem_u32(KG), vb = smem_u32(VG), pb = smem_u32(Ps);
        const uint32_t pkb = smem_u32(PKs), pvb = smem_u32(PVs);
        const uint32_t hs = (uint32_t)f.R * 128;
        for (int t = 0; t < ntiles && go; ++t) {
          const uint32_t Tt = T + t;
          go = mbar_wait(q_full, Tt & 1u, a.status);
          if (!go) break;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = tc::desc_kmajor_sw128(qb + (kk >> 2) * kHalf + (kk & 3) * 32);
            tc::mma_bf16(tmem, ad, tc::desc_kmajor_sw128(kb + (kk >> 2) * hs + (kk & 3) * 32), idS, kk > 0);
            tc::mma_bf16(tmem + 256, ad, tc::desc_kmajor_sw128(pkb + (kk >> 2) * 2048 + (kk & 3) * 32), idP,
                         kk > 0);
          }
          tc::mma_commit(s_full);
          go = mbar_wait(p_full, Tt & 1u, a.status);
          if (go && Tt > 0) go = mbar_wait(o_free, (Tt - 1) & 1u, a.status);
          if (!go) break;
          tc::fence_after_sync();
          for (int kk = 0; kk < n16 / 16; ++kk)
            tc::mma_bf16(tmem + 384, tc::desc_kmajor_sw128(pb + (kk >> 2) * kHalf + (kk & 3) * 32),
                         tc::desc_mnmajor_sw128(vb + kk * 2048, hs), idO, kk > 0);
          {
            const int kk = n16 / 16;  // the coarse pages' weights and mean values
            tc::mma_bf16(tmem + 384, tc::desc_kmajor_sw128(pb + (kk >> 2) * kHalf + (kk & 3) * 32),
                         tc::desc_mnmajor_sw128(pvb, 2048), idO, true);
          }
          tc::mma_commit(o_done);
        }
        if (!go) set_status(a.status, LOD_ST_TIMEOUT);
      }
      __syncwarp();
    } else {
      // ============================================================ pairs
      const int q4 = warp & 3;
      const int r = 32 * q4 + lane;
      const uint32_t tl = (uint32_t)(32 * q4) << 16;
      // the query row of pair t * 128 + r, staged by this thread
      auto gather = [&](int t, int64_t& pid) {
        const int idx = t * kRows + r;
        const bool v = idx < f.count;
        pid = v ? a.list[f.start + idx] : -1;
        const __nv_bfloat16* src = a.q;
        if (v) {
          const int64_t wr = pid / G;
          const int64_t bh = wr / a.NW, pi = a.w_lo + wr % a.NW;
          src = a.q + (bh * a.Tq + pi) * D;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c)
          cp_async16_zfill(Qs + (c >> 3) * kHalf + sw_off(r, c), reinterpret_cast<const uint4*>(src) + c, v);
        cp_async_mbar_arrive_noinc(q_full);
      };
      int64_t pid_cur = -1, pid_next = -1;
      gather(0, pid_cur);
      // page counts of the group (log2, for the coarse logits)
      if (r < 16) {
        float v = -INFINITY;
        if (f.ok && r < f.np) {
          const int pc = a.pCnt[(f.u * a.Cmax + f.c) * a.P + f.p0 + r];
          if (pc > 0 && pc <= kPage) v = log2f((float)pc);
          else set_status(a.status, LOD_ST_BAD_COUNT);
        }
        lpc_s[r] = v;
      }
      // rows past the group's members, and page slots past its pages, are
      // not inputs of this group: zero their values for MMA 2
      alive = mbar_wait(gfull, ngrp & 1u, a.status);
      if (alive) {
        const int hs = f.R * 128;
        for (int x = r; x < (n16 - f.n) * 16; x += 128) {
          const int row = f.n + x / 16, ch = x % 16;
          *reinterpret_cast<uint4*>(VG + (ch >> 3) * hs + sw_off(row, ch)) = make_uint4(0, 0, 0, 0);
        }
        for (int x = r; x < (16 - f.np) * 16; x += 128) {
          const int row = f.np + x / 16, ch = x % 16;
          *reinterpret_cast<uint4*>(PVs + (ch >> 3) * 2048 + sw_off(row, ch)) = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async();
      }
      bar_named_sync(kBarSoftB, 128);
      for (int t = 0; t < ntiles && alive; ++t) {
        const uint32_t Tt = T + t;
        alive = __all_sync(0xffffffffu, mbar_wait(s_full, Tt & 1u, a.status));
        if (!alive) break;
        tc::fence_after_sync();
        if (t + 1 < ntiles && !f.shared_qp) gather(t + 1, pid_next);
        // page scores and this row's top-TP pages (score desc, slot asc)
        float sp[16];
        tc::tmem_ld16(tmem + tl + 256, sp);
        uint32_t selm = 0;
        if (TP == 0 || TP >= f.np) {
          selm = (1u << f.np) - 1u;
        } else {
#pragma unroll
          for (int x = 0; x < kMaxTopPages; ++x) {
            if (x < TP) {
              float bs = -INFINITY;
              int bj = -1;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < f.np && !((selm >> j) & 1u) && (bj < 0 || sp[j] > bs)) {
                  bs = sp[j];
                  bj = j;
                }
              selm |= 1u << bj;
            }
          }
        }
        // pass 1: the row's max over its exact members and coarse pages
        float xc[16];
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool coarse = TP > 0 && j < f.np && !((selm >> j) & 1u);
          xc[j] = coarse ? fmaf(sp[j], scl, lpc_s[j]) : -INFINITY;
          m = fmaxf(m, xc[j]);
        }
        for (int j = 0; j < f.np; ++j) {
          float v[16];
          tc::tmem_ld16(tmem + tl + 16 * j, v);
          if ((selm >> j) & 1u) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (16 * j + e < f.n) m = fmaxf(m, v[e] * scl);
          }
        }
        const float mu = m == -INFINITY ? 0.f : m;
        // pass 2: the weights into P (members, then the coarse pages)
        float l = 0.f;
        for (int j = 0; j < f.np; ++j) {
          float v[16];
          tc::tmem_ld16(tmem + tl + 16 * j, v);
          const bool on = (selm >> j) & 1u;
          float p[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            p[e] = (on && 16 * j + e < f.n) ? ex2_approx(fmaf(v[e], scl, -mu)) : 0.f;
            l += p[e];
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ch = 2 * j + h;
            *reinterpret_cast<uint4*>(Ps + (ch >> 3) * kHalf + sw_off(r, ch)) =
                make_uint4(pack_bf16x2(p[8 * h], p[8 * h + 1]), pack_bf16x2(p[8 * h + 2], p[8 * h + 3]),
                           pack_bf16x2(p[8 * h + 4], p[8 * h + 5]), pack_bf16x2(p[8 * h + 6], p[8 * h + 7]));
          }
        }
        {
          float p[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            p[e] = xc[e] == -INFINITY ? 0.f : ex2_approx(xc[e] - mu);
            l += p[e];
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ch = n16 / 8 + h;
            *reinterpret_cast<uint4*>(Ps + (ch >> 3) * kHalf + sw_off(r, ch)) =
                make_uint4(pack_bf16x2(p[8 * h], p[8 * h + 1]), pack_bf16x2(p[8 * h + 2], p[8 * h + 3]),
                           pack_bf16x2(p[8 * h + 4], p[8 * h + 5]), pack_bf16x2(p[8 * h + 6], p[8 * h + 7]));
          }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // ---- epilogue: the pair's normalised partial
        alive = __all_sync(0xffffffffu, mbar_wait(o_done, Tt & 1u, a.status));
        if (!alive) break;
        tc::fence_after_sync();
        const bool vp = pid_cur >= 0 && f.ok;
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float ov[32];
          tc::tmem_ld32(tmem + tl + 384 + 32 * c, ov);
          if (vp) {
            uint4* dst = reinterpret_cast<uint4*>(a.po + pid_cur * D + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(ov[8 * q] * inv, ov[8 * q + 1] * inv),
                                  pack_bf16x2(ov[8 * q + 2] * inv, ov[8 * q + 3] * inv),
                                  pack_bf16x2(ov[8 * q + 4] * inv, ov[8 * q + 5] * inv),
                                  pack_bf16x2(ov[8 * q + 6] * inv, ov[8 * q + 7] * inv));
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
        if (pid_cur >= 0) {
          a.plse[pid_cur] = vp && l > 0.f ? m + log2f(l) : -INFINITY;
          if (a.sel_pages) {
            const int64_t wr = pid_cur / G;
            const int rank = (int)(pid_cur % G);
            const int64_t bh = wr / a.NW, pi = a.w_lo + wr % a.NW;
            int32_t* spo = a.sel_pages + ((bh * a.Tq + pi) * G + rank) * TP;
            // the opened pages, best first (score desc, slot asc)
            uint32_t rest = vp ? selm : 0u;
            for (int x = 0; x < TP; ++x) {
              int bj = -1;
              float bs = -INFINITY;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (((rest >> j) & 1u) && (bj < 0 || sp[j] > bs)) {
                  bs = sp[j];
                  bj = j;
                }
              spo[x] = bj >= 0 ? (int32_t)(f.c * a.P + f.p0 + bj) : -1;
              if (bj >= 0) rest &= ~(1u << bj);
            }
          }
        }
        if (t + 1 < ntiles && f.shared_qp) gather(t + 1, pid_next);
        pid_cur = pid_next;
      }
      // (a gathered tile that was never consumed: let its copies land)
      cp_async_wait_all();
    }
    T += (uint32_t)ntiles;
    ++ngrp;
    alive = !__syncthreads_or(!alive);
  }
  if (!alive && tid == 0) set_status(a.status, LOD_ST_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ================================================================== merge

// One warp per row: the row state (m, l, acc) and the partials of the
// row's opened groups in one softmax.
__global__ void __launch_bounds__(256) pf_merge_kernel(const __grid_constant__ PrefillArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.NW;
  const int64_t wr = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wr >= nrows) return;
  const int64_t bh = wr / a.NW, pi = a.w_lo + wr % a.NW;
  if (pi >= a.w_hi) return;
  const int64_t orow = bh * a.Tq + pi;
  const float* stp = a.state + wr * kStateStride;
  const float m = stp[0], l = stp[1];
  // (a row whose scan gave up holds m = -inf and no accumulator)
  const float4 acc = m == -INFINITY ? make_float4(0.f, 0.f, 0.f, 0.f)
                                    : *reinterpret_cast<const float4*>(stp + 4 + 4 * lane);
  float M = m;
  for (int k = 0; k < a.G; ++k)
    if (a.sel[wr * a.G + k] >= 0) M = fmaxf(M, a.plse[wr * a.G + k]);
  const float cs = m == -INFINITY ? 0.f : ex2_approx(m - M);
  float L = l * cs;
  float o0 = acc.x * cs, o1 = acc.y * cs, o2 = acc.z * cs, o3 = acc.w * cs;
  for (int k = 0; k < a.G; ++k) {
    if (a.sel[wr * a.G + k] < 0) {
      if (a.sel_pages && lane < a.TP) a.sel_pages[(orow * a.G + k) * a.TP + lane] = -1;
      continue;
    }
    const float ls = a.plse[wr * a.G + k];
    if (ls == -INFINITY) continue;
    const float w = ex2_approx(ls - M);
    L += w;
    const uint2 raw = *reinterpret_cast<const uint2*>(a.po + (wr * a.G + k) * D + 4 * lane);
    o0 = fmaf(w, __uint_as_float(raw.x << 16), o0);
    o1 = fmaf(w, __uint_as_float(raw.x & 0xffff0000u), o1);
    o2 = fmaf(w, __uint_as_float(raw.y << 16), o2);
    o3 = fmaf(w, __uint_as_float(raw.y & 0xffff0000u), o3);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  *reinterpret_cast<uint2*>(a.out + orow * D + 4 * lane) =
      make_uint2(pack_bf16x2(o0 * inv, o1 * inv), pack_bf16x2(o2 * inv, o3 * inv));
  if (lane == 0 && a.lse) a.lse[orow] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace

size_t prefill_tc_scan_smem() { return SmemA::bytes; }
size_t prefill_tc_pair_smem() { return SmemB::bytes; }

cudaError_t launch_prefill_tc_wave(const PrefillArgs& a, const TcMaps& maps, const PairMaps& pmaps, int num_sms,
                                   cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * (size_t)a.Gtot, stream);
  if (e != cudaSuccess) return e;
  const int RP = kRows / a.g;
  const int64_t nblk = (a.w_hi - a.w_lo + RP - 1) / RP;
  const int64_t tiles = nblk * a.B * a.Hkv;
  if (a.G <= 8) {
    e = set_smem_once<pf_scan_kernel<8>>(SmemA::bytes);
    if (e == cudaSuccess)
      pf_scan_kernel<8><<<(unsigned)tiles, kThreadsA, SmemA::bytes, stream>>>(maps, a);
  } else {
    e = set_smem_once<pf_scan_kernel<16>>(SmemA::bytes);
    if (e == cudaSuccess)
      pf_scan_kernel<16><<<(unsigned)tiles, kThreadsA, SmemA::bytes, stream>>>(maps, a);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pf_plan_kernel<<<1, kPlanThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t npairs = (int64_t)a.B * a.Hq * a.NW * a.G;
  const int64_t sblocks = (npairs + 255) / 256 < 4 * num_sms ? (npairs + 255) / 256 : 4 * num_sms;
  pf_scatter_kernel<<<(unsigned)(sblocks > 0 ? sblocks : 1), 256, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = set_smem_once<pf_pair_kernel>(SmemB::bytes);
  if (e != cudaSuccess) return e;
  pf_pair_kernel<<<(unsigned)num_sms, kThreadsB, SmemB::bytes, stream>>>(pmaps, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hq * a.NW;
  pf_merge_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace lod
