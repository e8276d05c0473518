// lod_build.cu -- online multi-resolution index build ("Level of Detail
// Attention", How It Works, paragraph 1): per 256-token chunk, k-means groups,
// 16-key pages, and their mean keys, mean values and counts.
//
// One CTA of 256 threads per (chunk, KV head, sequence); thread i owns the
// chunk's i-th clustered key and keeps it in registers as fp32.  Centroids
// live in shared memory and are read as warp-uniform (broadcast) float4
// loads, so the assignment step is one FMA per (key, centroid, dimension)
// in the expanded form ||c||^2 - 2 k.c (the ||k||^2 term is common to all
// centroids of a key and cannot change its argmin).
//
// The update step is deterministic: members are counting-sorted by cluster
// (stable, ascending position) and every (cluster, dimension) sum is taken by
// one thread in that order.  Hence an iteration whose assignment equals the
// previous one reproduces the previous centroids bit for bit, every later
// round would repeat it, and the loop may stop there with an unchanged
// result.
#include "lod_internal.cuh"

namespace lod {

namespace {

constexpr int kBuildThreads = 256;

template <int N>
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
    v = lane < N ? red_s[lane] : -INFINITY;
    idx = lane < N ? red_i[lane] : 0x7fffffff;
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
      red_s[N] = v;
      red_i[N] = idx;
    }
  }
  __syncthreads();
  out_v = red_s[N];
  out_i = red_i[N];
  __syncthreads();
}

template <typename T, int D, int KMAX>
__global__ void __launch_bounds__(kBuildThreads, 1) kmeans_kernel(BuildArgs a) {
  constexpr int NW = kBuildThreads / 32;
  constexpr int ROW_BYTES = D * (int)sizeof(T) + 16;  // padded row: conflict-free per-thread rows
  const int64_t c = a.chunk_begin + blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t unit = (int64_t)b * a.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int first = (c == 0) ? a.sinks : 0;  // sink positions are never clustered
  const int n = kChunk - first;
  const int k = a.k;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* cen = reinterpret_cast<float*>(smem_raw);              // [KMAX][D]
  float* cnorm = cen + KMAX * D;                                // [KMAX]
  float* red_s = cnorm + KMAX;                                  // [NW + 1]
  int* red_i = reinterpret_cast<int*>(red_s + NW + 1);          // [NW + 1]
  int* wcnt = red_i + NW + 1;                                   // [NW][KMAX]
  int* cnt = wcnt + NW * KMAX;                                  // [KMAX]
  int* off = cnt + KMAX;                                        // [KMAX + 1]
  int* pstart = off + KMAX + 1;                                 // [KMAX + 1]
  int* perm_s = pstart + KMAX + 1;                              // [kChunk]
  unsigned char* xs = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(perm_s + kChunk) + 15) & ~uintptr_t(15));  // [kChunk][ROW_BYTES]

  const T* Kc = static_cast<const T*>(a.K) + b * a.sb + h * a.sh + c * kChunk * a.st;
  const T* Vc = static_cast<const T*>(a.V) + b * a.sb + h * a.sh + c * kChunk * a.st;

  // ---- own key into registers (fp32) and into the padded shared-memory copy
  float x[D];
  if (tid < n) {
    const T* row = Kc + (int64_t)(first + tid) * a.st;
    constexpr int VEC = 16 / sizeof(T);
#pragma unroll
    for (int i = 0; i < D; i += VEC) {
      uint4 raw = __ldg(reinterpret_cast<const uint4*>(row + i));
      *reinterpret_cast<uint4*>(xs + tid * ROW_BYTES + i * sizeof(T)) = raw;
      float f[VEC];
      load_f<T, VEC>(row + i, f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) x[i + e] = f[e];
    }
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) x[i] = 0.f;
  }

  // ---- seeded farthest-first initialisation
  float mind = tid < n ? INFINITY : -INFINITY;
  for (int j = 0; j < k; ++j) {
    int pick;
    if (j == 0) {
      const uint64_t hsh = splitmix64(a.seed ^ ((uint64_t(unit) << 32) + uint64_t(c)));
      pick = (int)(hsh % uint64_t(n));
    } else {
      float bv;
      block_argmax<NW>(tid < n ? mind : -INFINITY, tid, red_s, red_i, bv, pick);
    }
    if (tid == pick) {
#pragma unroll
      for (int i = 0; i < D; ++i) cen[j * D + i] = x[i];
    }
    __syncthreads();
    if (tid < n) {
      float dd = 0.f;
#pragma unroll
      for (int i = 0; i < D; i += 4) {
        float4 cc = *reinterpret_cast<const float4*>(cen + j * D + i);
        float t0 = x[i] - cc.x, t1 = x[i + 1] - cc.y, t2 = x[i + 2] - cc.z, t3 = x[i + 3] - cc.w;
        dd = fmaf(t0, t0, dd);
        dd = fmaf(t1, t1, dd);
        dd = fmaf(t2, t2, dd);
        dd = fmaf(t3, t3, dd);
      }
      mind = fminf(mind, dd);
    }
  }
  // centroid norms
  for (int j = warp; j < k; j += NW) {
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s = fmaf(cen[j * D + i], cen[j * D + i], s);
    s = warp_sum(s);
    if (lane == 0) cnorm[j] = s;
  }
  __syncthreads();

  // ---- Lloyd rounds
  int a_prev = -1;
  for (int it = 0; it < a.iters; ++it) {
    int a_new = 0;
    if (tid < n) {
      float dot[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) dot[j] = 0.f;
#pragma unroll
      for (int i = 0; i < D; i += 4) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (j < k) {
            float4 cc = *reinterpret_cast<const float4*>(cen + j * D + i);
            dot[j] = fmaf(x[i], cc.x, dot[j]);
            dot[j] = fmaf(x[i + 1], cc.y, dot[j]);
            dot[j] = fmaf(x[i + 2], cc.z, dot[j]);
            dot[j] = fmaf(x[i + 3], cc.w, dot[j]);
          }
        }
      }
      float best = fmaf(-2.f, dot[0], cnorm[0]);
#pragma unroll
      for (int j = 1; j < KMAX; ++j) {
        if (j < k) {
          float dj = fmaf(-2.f, dot[j], cnorm[j]);
          if (dj < best) {  // strict: ties keep the lower cluster id
            best = dj;
            a_new = j;
          }
        }
      }
    }
    const int changed = __syncthreads_or(tid < n && a_new != a_prev);
    if (it > 0 && !changed) break;  // fixed point: later rounds repeat this one exactly
    a_prev = a_new;

    // stable counting sort of members by cluster (ascending local index)
    int rank = 0;
    for (int j = 0; j < k; ++j) {
      unsigned m = __ballot_sync(0xffffffffu, tid < n && a_new == j);
      if (lane == 0) wcnt[warp * KMAX + j] = __popc(m);
      if (tid < n && a_new == j) rank = __popc(m & ((1u << lane) - 1u));
    }
    __syncthreads();
    if (tid == 0) {
      int o = 0;
      for (int j = 0; j < k; ++j) {
        off[j] = o;
        int cj = 0;
        for (int w = 0; w < NW; ++w) {
          int t = wcnt[w * KMAX + j];
          wcnt[w * KMAX + j] = o + cj;  // becomes the warp's base offset for cluster j
          cj += t;
        }
        cnt[j] = cj;
        o += cj;
      }
      off[k] = o;
    }
    __syncthreads();
    if (tid < n) perm_s[wcnt[warp * KMAX + a_new] + rank] = tid;
    __syncthreads();

    // centroid := member mean (fp32, ascending member order); empty clusters keep theirs
    for (int item = tid; item < k * D; item += kBuildThreads) {
      const int j = item / D, i = item % D;
      const int cj = cnt[j];
      if (cj > 0) {
        float s = 0.f;
        for (int m = off[j]; m < off[j] + cj; ++m)
          s += Elem<T>::to_f(*reinterpret_cast<const T*>(xs + perm_s[m] * ROW_BYTES + i * sizeof(T)));
        cen[j * D + i] = s / (float)cj;
      }
    }
    __syncthreads();
    for (int j = warp; j < k; j += NW) {
      float s = 0.f;
      for (int i = lane; i < D; i += 32) s = fmaf(cen[j * D + i], cen[j * D + i], s);
      s = warp_sum(s);
      if (lane == 0) cnorm[j] = s;
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
  if (tid < k) gCnt[tid] = cnt[tid];
  if (tid < P) {
    int used = pstart[k];
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

  // summaries: one thread per (group, dimension, K-or-V), fp32 sums in member order
  for (int item = tid; item < 2 * k * D; item += kBuildThreads) {
    const int isv = item / (k * D);
    const int j = (item / D) % k, i = item % D;
    const int cj = cnt[j];
    T* gdst = isv ? gV : gK;
    T* pdst = isv ? pV : pK;
    if (cj == 0) {
      gdst[j * D + i] = Elem<T>::from_f(0.f);
      continue;
    }
    float gs = 0.f, ps = 0.f;
    int inpage = 0, slot = pstart[j];
    for (int m = off[j]; m < off[j] + cj; ++m) {
      const int loc = perm_s[m];
      float v = isv ? Elem<T>::to_f(Vc[(int64_t)(first + loc) * a.st + i])
                    : Elem<T>::to_f(*reinterpret_cast<const T*>(xs + loc * ROW_BYTES + i * sizeof(T)));
      gs += v;
      ps += v;
      if (++inpage == kPage) {
        pdst[slot * D + i] = Elem<T>::from_f(ps / (float)kPage);
        ++slot;
        ps = 0.f;
        inpage = 0;
      }
    }
    if (inpage > 0) pdst[slot * D + i] = Elem<T>::from_f(ps / (float)inpage);
    // the group key mean is the final centroid: the same fp32 sum / count
    gdst[j * D + i] = Elem<T>::from_f(isv ? gs / (float)cj : cen[j * D + i]);
  }
  // unused page slots hold zeros
  for (int item = tid; item < (int)(P - pstart[k]) * D; item += kBuildThreads) {
    const int slot = pstart[k] + item / D, i = item % D;
    pK[slot * D + i] = Elem<T>::from_f(0.f);
    pV[slot * D + i] = Elem<T>::from_f(0.f);
  }
}

template <int D, int KMAX>
size_t kmeans_smem_bytes(size_t elem) {
  constexpr int NW = kBuildThreads / 32;
  size_t s = sizeof(float) * (KMAX * D + KMAX + NW + 1) + sizeof(int) * (NW + 1 + NW * KMAX + KMAX +
                                                                          2 * (KMAX + 1) + kChunk);
  s = (s + 15) & ~size_t(15);
  s += (size_t)kChunk * (D * elem + 16);
  return s;
}

template <typename T, int D, int KMAX>
cudaError_t launch_kmeans_t(const BuildArgs& a, int64_t nchunks, int B, cudaStream_t stream) {
  const size_t smem = kmeans_smem_bytes<D, KMAX>(sizeof(T));
  auto kern = kmeans_kernel<T, D, KMAX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
