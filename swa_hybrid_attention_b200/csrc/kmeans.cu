// k-means clustering of the projected keys of a KV cache.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": after the
// low-rank projection, semantically related keys lie close together, so
// clustering them ("聚类中心") lets whole groups of unrelated tokens be skipped;
// the page's deployment runs full attention in prefill, clusters the K cache
// and decodes sparsely.  The library reads the clustering as Lloyd's k-means
// on the 16-dim projected keys X_j = P^T k_j of rows [block, clu_end) of every
// retrieval head (the sink block and the unclustered tail are attended in
// full by the decode step):
//   seeds     mu_c = X[floor((2c+1) n / (2 nc))]
//   each of `iters` rounds: assign every key to the nearest centroid
//             (ties to the lower index), then move each centroid to the mean
//             of its keys (an empty cluster keeps its centroid).
// The distance is evaluated as |mu|^2 - 2 x.mu (|x|^2 is common to all
// centroids of a key).  Every sum has a fixed order and the grouping of keys
// by cluster is a stable counting sort, so results are bit-reproducible.
//
// Kernels (retrieval heads only; CTAs of other heads leave at once):
//   km_project    one thread per key: X = P^T k (fixed order over d)
//   km_seed       the evenly spaced seeds
//   km_assign     four keys per thread against every centroid, the centroids
//                 in shared memory
//   km_group      one CTA of 1024 threads per (sequence, head): cluster sizes,
//                 offsets (scan), stable placement of the keys (one warp,
//                 32 keys per step with match_any), and the new centroids
//                 (each summed over its keys in position order)
//   km_chunks     each cluster's keys cut into chunks of <= 128 (the units
//                 the decode step selects), with the cluster's centroid
//   km_permute    K and V rows copied into cluster order (one warp per row;
//                 skipped when the caller asks for no copy: the decode then
//                 gathers member rows in place)

#include <cuda_bf16.h>

#include "internal.cuh"

namespace rtp {
namespace {

constexpr int kKmThreads = 256;
constexpr int kGroupThreads = 1024;

__device__ __forceinline__ size_t head_index(const KmeansArgs& a) {
  return static_cast<size_t>(blockIdx.z) * a.n_kv_heads + blockIdx.y;
}

__global__ void __launch_bounds__(kKmThreads) km_project_kernel(const KmeansArgs a) {
  __shared__ float P[kHeadDim * kRank];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  for (int e = threadIdx.x; e < kHeadDim * kRank; e += kKmThreads) P[e] = a.proj[e];
  __syncthreads();
  const int j = blockIdx.x * kKmThreads + threadIdx.x;
  if (j >= a.n) return;
  const size_t bk = head_index(a);
  const uint4* row = reinterpret_cast<const uint4*>(
      a.kcache + (bk * a.cache_cap + a.block + static_cast<size_t>(j)) * kHeadDim);
  float acc[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) acc[c] = 0.f;
  for (int d8 = 0; d8 < kHeadDim / 8; ++d8) {
    const uint4 u = row[d8];
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      const float* p0 = P + (8 * d8 + 2 * e) * kRank;
#pragma unroll
      for (int c = 0; c < kRank; ++c) acc[c] = fmaf(f.x, p0[c], acc[c]);
#pragma unroll
      for (int c = 0; c < kRank; ++c) acc[c] = fmaf(f.y, p0[kRank + c], acc[c]);
    }
  }
  float4* out = reinterpret_cast<float4*>(a.X + (bk * a.n + j) * kRank);
#pragma unroll
  for (int w = 0; w < 4; ++w) out[w] = make_float4(acc[4 * w], acc[4 * w + 1], acc[4 * w + 2], acc[4 * w + 3]);
}

__global__ void __launch_bounds__(kKmThreads) km_seed_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  for (int e = threadIdx.x; e < a.nc * kRank; e += kKmThreads) {
    const int c = e / kRank, d = e % kRank;
    const long j = (static_cast<long>(2 * c + 1) * a.n) / (2L * a.nc);
    a.centroids[(bk * a.nc + c) * kRank + d] = a.X[(bk * a.n + j) * kRank + d];
  }
}

// Keys per thread in km_assign: every centroid read from shared memory
// serves this many keys (the loop is bound by shared-memory loads otherwise).
constexpr int kAssignKeys = 4;

__global__ void __launch_bounds__(kKmThreads) km_assign_kernel(const KmeansArgs a) {
  extern __shared__ float4 mu4[];  // [nc][4] centroids, then [nc] squared norms
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  float* nrm = reinterpret_cast<float*>(mu4 + 4 * a.nc);
  const float4* src = reinterpret_cast<const float4*>(a.centroids + bk * a.nc * kRank);
  for (int e = threadIdx.x; e < 4 * a.nc; e += kKmThreads) mu4[e] = src[e];
  __syncthreads();
  for (int c = threadIdx.x; c < a.nc; c += kKmThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 m = mu4[4 * c + w];
      s = fmaf(m.x, m.x, s);
      s = fmaf(m.y, m.y, s);
      s = fmaf(m.z, m.z, s);
      s = fmaf(m.w, m.w, s);
    }
    nrm[c] = s;
  }
  __syncthreads();
  // keys j0 + u * kKmThreads, u < kAssignKeys (coalesced over the CTA)
  const int j0 = blockIdx.x * kKmThreads * kAssignKeys + threadIdx.x;
  float x[kAssignKeys][kRank];
#pragma unroll
  for (int u = 0; u < kAssignKeys; ++u) {
    const int j = min(j0 + u * kKmThreads, a.n - 1);
    const float4* xr = reinterpret_cast<const float4*>(a.X + (bk * a.n + j) * kRank);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 v = xr[w];
      x[u][4 * w] = v.x;
      x[u][4 * w + 1] = v.y;
      x[u][4 * w + 2] = v.z;
      x[u][4 * w + 3] = v.w;
    }
  }
  float best[kAssignKeys];
  int bc[kAssignKeys];
#pragma unroll
  for (int u = 0; u < kAssignKeys; ++u) {
    best[u] = INFINITY;
    bc[u] = 0;
  }
  for (int c = 0; c < a.nc; ++c) {
    const float4 m0 = mu4[4 * c], m1 = mu4[4 * c + 1], m2 = mu4[4 * c + 2], m3 = mu4[4 * c + 3];
    const float nc2 = nrm[c];
    const float m[kRank] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w,
                            m2.x, m2.y, m2.z, m2.w, m3.x, m3.y, m3.z, m3.w};
#pragma unroll
    for (int u = 0; u < kAssignKeys; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int d = 0; d < kRank; ++d) dot = fmaf(x[u][d], m[d], dot);
      const float dist = fmaf(-2.f, dot, nc2);
      if (dist < best[u]) {
        best[u] = dist;
        bc[u] = c;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kAssignKeys; ++u) {
    const int j = j0 + u * kKmThreads;
    if (j < a.n) a.assign[bk * a.n + j] = bc[u];
  }
}

// Exclusive scan of v over the CTA (kGroupThreads threads, thread order).
__device__ __forceinline__ int cta_exclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    warp_tot[lane] = wi - w;
  }
  __syncthreads();
  const int r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

// Offsets of nc counts (exclusive scan); each thread takes two consecutive
// clusters (nc <= 2 * kGroupThreads).
__device__ __forceinline__ void scan_counts(const int* cnt, int* off, int nc, int* warp_tot) {
  const int c0 = 2 * threadIdx.x;
  const int v0 = c0 < nc ? cnt[c0] : 0, v1 = c0 + 1 < nc ? cnt[c0 + 1] : 0;
  const int base = cta_exclusive_scan(v0 + v1, warp_tot);
  if (c0 < nc) off[c0] = base;
  if (c0 + 1 < nc) off[c0 + 1] = base + v0;
}

__global__ void __launch_bounds__(kGroupThreads) km_group_kernel(const KmeansArgs a) {
  __shared__ int cnt[kMaxClusters], off[kMaxClusters], running[kMaxClusters];
  __shared__ int warp_tot[32];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int tid = threadIdx.x, lane = tid & 31;
  const int32_t* asg = a.assign + bk * a.n;
  for (int c = tid; c < a.nc; c += kGroupThreads) {
    cnt[c] = 0;
    running[c] = 0;
  }
  __syncthreads();
  for (int j = tid; j < a.n; j += kGroupThreads) atomicAdd(&cnt[asg[j]], 1);
  __syncthreads();
  scan_counts(cnt, off, a.nc, warp_tot);
  __syncthreads();
  int32_t* offs = a.offsets + bk * (a.nc + 1);
  for (int c = tid; c < a.nc; c += kGroupThreads) offs[c] = off[c];
  if (tid == 0) offs[a.nc] = a.n;
  // stable placement: one warp walks the keys in order, 32 at a time
  int32_t* mem = a.members + bk * a.n;
  if (tid < 32) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < a.n; j0 += 32 * 8) {
      int cj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + 32 * u + lane;
        cj[u] = j < a.n ? asg[j] : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = cj[u];
        const uint32_t peers = __match_any_sync(0xffffffffu, c);
        if (c >= 0) mem[off[c] + running[c] + __popc(peers & lt)] = a.block + j0 + 32 * u + lane;
        __syncwarp();
        if (c >= 0 && lane == __ffs(peers) - 1) running[c] += __popc(peers);
        __syncwarp();
      }
    }
  }
  __syncthreads();
  // new centroids: the mean of each cluster's keys, summed in position order
  for (int c = tid; c < a.nc; c += kGroupThreads) {
    const int size = cnt[c];
    if (size == 0) continue;
    float s[kRank];
#pragma unroll
    for (int d = 0; d < kRank; ++d) s[d] = 0.f;
    for (int e = 0; e < size; ++e) {
      const int j = mem[off[c] + e] - a.block;
      const float4* xr = reinterpret_cast<const float4*>(a.X + (bk * a.n + j) * kRank);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 v = xr[w];
        s[4 * w] += v.x;
        s[4 * w + 1] += v.y;
        s[4 * w + 2] += v.z;
        s[4 * w + 3] += v.w;
      }
    }
    float* mu = a.centroids + (bk * a.nc + c) * kRank;
#pragma unroll
    for (int d = 0; d < kRank; ++d) mu[d] = s[d] / static_cast<float>(size);
  }
}

__global__ void __launch_bounds__(kGroupThreads) km_chunks_kernel(const KmeansArgs a) {
  __shared__ int nch[kMaxClusters], choff[kMaxClusters];
  __shared__ int warp_tot[32];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int tid = threadIdx.x;
  const int32_t* offs = a.offsets + bk * (a.nc + 1);
  for (int c = tid; c < a.nc; c += kGroupThreads) nch[c] = (offs[c + 1] - offs[c] + 127) / 128;
  __syncthreads();
  scan_counts(nch, choff, a.nc, warp_tot);
  __syncthreads();
  const size_t base = bk * a.max_chunks;
  for (int c = tid; c < a.nc; c += kGroupThreads) {
    const int size = offs[c + 1] - offs[c];
    const float4* mu = reinterpret_cast<const float4*>(a.centroids + (bk * a.nc + c) * kRank);
    for (int m = 0; m < nch[c]; ++m) {
      const size_t id = base + choff[c] + m;
      a.chunk_start[id] = offs[c] + 128 * m;
      a.chunk_len[id] = min(128, size - 128 * m);
      float4* cc = reinterpret_cast<float4*>(a.chunk_centroids + id * kRank);
#pragma unroll
      for (int w = 0; w < 4; ++w) cc[w] = mu[w];
    }
  }
  if (tid == kGroupThreads - 1) a.n_chunks[bk] = choff[a.nc - 1] + nch[a.nc - 1];
}

__global__ void __launch_bounds__(kKmThreads) km_permute_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int r = blockIdx.x * (kKmThreads / 32) + (threadIdx.x >> 5);
  if (r >= a.n) return;
  const int lane = threadIdx.x & 31;
  const int src = a.members[bk * a.n + r];
  const bool is_v = lane >= 16;
  const uint4* from = reinterpret_cast<const uint4*>((is_v ? a.vcache : a.kcache) +
                                                     (bk * a.cache_cap + static_cast<size_t>(src)) * kHeadDim);
  uint4* to = reinterpret_cast<uint4*>((is_v ? a.v_sorted : a.k_sorted) + (bk * a.n + r) * kHeadDim);
  to[lane & 15] = from[lane & 15];
}

}  // namespace

cudaError_t launch_kmeans(const KmeansArgs& a, int iters, cudaStream_t stream) {
  const dim3 per_key((a.n + kKmThreads - 1) / kKmThreads, a.n_kv_heads, a.batch);
  const dim3 per_keys((a.n + kKmThreads * kAssignKeys - 1) / (kKmThreads * kAssignKeys), a.n_kv_heads, a.batch);
  const dim3 per_head(1, a.n_kv_heads, a.batch);
  km_project_kernel<<<per_key, kKmThreads, 0, stream>>>(a);
  km_seed_kernel<<<per_head, kKmThreads, 0, stream>>>(a);
  const size_t smem = static_cast<size_t>(a.nc) * (kRank + 1) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(km_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  for (int it = 0; it < iters; ++it) {
    km_assign_kernel<<<per_keys, kKmThreads, smem, stream>>>(a);
    km_group_kernel<<<per_head, kGroupThreads, 0, stream>>>(a);
  }
  km_chunks_kernel<<<per_head, kGroupThreads, 0, stream>>>(a);
  if (a.k_sorted) {  // no cluster-ordered copy when the decode reads member rows in place
    const dim3 per_row((a.n + kKmThreads / 32 - 1) / (kKmThreads / 32), a.n_kv_heads, a.batch);
    km_permute_kernel<<<per_row, kKmThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace rtp
