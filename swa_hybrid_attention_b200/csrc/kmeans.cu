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
//   km_assign_mma the distances of 32 keys per warp to every centroid by
//                 mma.sync (fp16 operands, fp32 accumulation, |mu|^2 as the
//                 accumulator's start); a key whose two smallest distances
//                 differ by more than twice the pass's proven error bound is
//                 assigned there, every other key is queued
//   km_rescore    the queued keys by the exact fp32 path (the same operations
//                 in the same order as km_assign, which does every key when
//                 RTP_KMEANS_EXACT_ASSIGN=1), so the assignment is the fp32
//                 path's, key for key
//   km_hist / km_segscan / km_scan / km_place / km_means  the keys grouped
//                 by cluster: per-segment counts, segment starts, offsets, stable
//                 placement (a warp per segment, 32 keys per step with
//                 match_any), and the new centroids (each summed over its
//                 keys in position order)
//   km_chunks     each cluster's keys cut into chunks of <= 128 (the units
//                 the decode step selects), with the cluster's centroid
//   km_permute    K and V rows copied into cluster order (one warp per row;
//                 skipped when the caller asks for no copy: the decode then
//                 gathers member rows in place)

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdlib>

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
  if (threadIdx.x == 0) a.amb_count[bk] = 0;
  for (int e = threadIdx.x; e < a.nc * kRank; e += kKmThreads) {
    const int c = e / kRank, d = e % kRank;
    const long j = (static_cast<long>(2 * c + 1) * a.n) / (2L * a.nc);
    a.centroids[(bk * a.nc + c) * kRank + d] = a.X[(bk * a.n + j) * kRank + d];
  }
}

// Keys per thread in km_assign: every centroid read from shared memory
// serves this many keys (the loop is bound by shared-memory loads otherwise).
constexpr int kAssignKeys = 4;

// The exact assignment: each key against every centroid in fp32 with the
// fixed operation order (|mu|^2 by fma over the 16 dims, x.mu by fma over
// the 16 dims, |mu|^2 - 2 x.mu, first minimum over ascending c).  Used for
// every key (km_assign_kernel) or for the keys the tensor-core pass could
// not decide (km_rescore_kernel); a key's result does not depend on which.
// kList: the CTA's keys are entries [first, first + kKmThreads*kAssignKeys)
// of the head's list of undecided keys (count entries); otherwise keys
// first + ... directly.
template <bool kList, int kThreads, int kKeys>
__device__ __forceinline__ void exact_assign(const KmeansArgs& a, size_t bk, int first, int count) {
  extern __shared__ float4 mu4[];  // [nc][4] centroids, then [nc] squared norms
  float* nrm = reinterpret_cast<float*>(mu4 + 4 * a.nc);
  const float4* src = reinterpret_cast<const float4*>(a.centroids + bk * a.nc * kRank);
  for (int e = threadIdx.x; e < 4 * a.nc; e += kThreads) mu4[e] = src[e];
  __syncthreads();
  for (int c = threadIdx.x; c < a.nc; c += kThreads) {
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
  // keys of entries e0 + u * kThreads, u < kKeys (coalesced over the CTA)
  const int e0 = first + threadIdx.x;
  int jk[kKeys];
#pragma unroll
  for (int u = 0; u < kKeys; ++u) {
    const int e = e0 + u * kThreads;
    jk[u] = e < count ? (kList ? a.amb_list[bk * a.n + e] : e) : -1;
  }
  float x[kKeys][kRank];
#pragma unroll
  for (int u = 0; u < kKeys; ++u) {
    const int j = min(max(jk[u], 0), a.n - 1);
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
  float best[kKeys];
  int bc[kKeys];
#pragma unroll
  for (int u = 0; u < kKeys; ++u) {
    best[u] = INFINITY;
    bc[u] = 0;
  }
  for (int c = 0; c < a.nc; ++c) {
    const float4 m0 = mu4[4 * c], m1 = mu4[4 * c + 1], m2 = mu4[4 * c + 2], m3 = mu4[4 * c + 3];
    const float nc2 = nrm[c];
    const float m[kRank] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w,
                            m2.x, m2.y, m2.z, m2.w, m3.x, m3.y, m3.z, m3.w};
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
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
  for (int u = 0; u < kKeys; ++u) {
    const int j = jk[u];
    if (j >= 0 && j < a.n) a.assign[bk * a.n + j] = bc[u];
  }
}

__global__ void __launch_bounds__(kKmThreads) km_assign_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  exact_assign<false, kKmThreads, kAssignKeys>(a, head_index(a), blockIdx.x * kKmThreads * kAssignKeys, a.n);
}

// gridDim.x CTAs per head walk the head's list in chunks of
// kKmThreads * kAssignKeys keys (the centroids are loaded once per chunk).
__global__ void __launch_bounds__(kKmThreads) km_rescore_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int count = min(a.amb_count[bk], a.n);
  for (int first = blockIdx.x * kKmThreads * kAssignKeys; first < count;
       first += gridDim.x * kKmThreads * kAssignKeys) {  // (uniform over the CTA)
    exact_assign<true, kKmThreads, kAssignKeys>(a, bk, first, count);
    __syncthreads();  // the shared centroids are loaded again for the next chunk
  }
}

// ------------------------------------------------ tensor-core assignment
// The distances of 16 keys to 8 centroids are one mma.sync m16n8k16: A = the
// keys' projections in fp16, B = -2 mu in fp16, C = |mu|^2 (fp32, the exact
// path's value), so D = |mu|^2 - 2 x~.mu~.  Each thread keeps, per key row,
// the smallest D, the group (four centroids of one tile pair) holding it and
// the smallest D among the other groups.  D differs from the exact path's fp32
// distance by at most
//   E = 1.125 * 2^-9 |x| M + 2^-16 M^2 + 2^-20 (|x| + M),   M = max_c |mu_c|
// (fp16 rounding of x and mu: 2^-11 relative each, products exact; fp32
// accumulation of 17 terms; the exact path's own fp32 rounding; with margin).
// A key whose other groups all lie more than 2E above its smallest D has the
// exact path's nearest centroid in its best group, found by the group's four
// exact distances (ascending, first minimum: the exact path's tie rule); every
// other key (and any key with non-finite values, |x| >= 30000 or M > 8192,
// outside fp16's safe range) is appended to the head's undecided list, which
// km_rescore_kernel assigns by the exact path.  The result is the exact
// path's, key for key.
constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = 32 * kMmaWarps;
constexpr int kMmaGroups = 4;                              // 32-key groups per warp
constexpr int kMmaKeysPerCta = kMmaThreads * kMmaGroups;  // 1024

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, float c0,
                                        float c1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void ldsm_x4_b16(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Running smallest distance m1 of one key row, the smallest distance L among
// the other groups (a group: the four centroids one thread sees in one
// 16-centroid tile pair) and the tile pair holding m1, updated with this
// thread's four distances of pair p: (d0, d1) from the first 8-centroid tile,
// (e0, e1) from the second.  If L exceeds m1 by more than twice the error
// bound, every centroid outside the group lies farther than the group's
// nearest, so the exact nearest centroid is one of the group's four.
__device__ __forceinline__ void top2_group(float& m1, float& L, int& pb, float d0, float d1, float e0, float e1,
                                           int p) {
  const float g1 = min3f(fminf(d0, d1), e0, e1);
  L = fminf(L, fmaxf(m1, g1));
  if (g1 < m1) pb = p;
  m1 = fminf(m1, g1);
}

// Merge with the quad neighbour at lane ^ mask (the same rows, other
// centroids, so other groups); owner = the quad lane whose group holds m1.
__device__ __forceinline__ void top2_merge(float& m1, float& L, int& pb, int& owner, int mask) {
  const float om1 = __shfl_xor_sync(0xffffffffu, m1, mask);
  const float oL = __shfl_xor_sync(0xffffffffu, L, mask);
  const int opb = __shfl_xor_sync(0xffffffffu, pb, mask);
  const int oown = __shfl_xor_sync(0xffffffffu, owner, mask);
  L = fminf(fmaxf(m1, om1), fminf(L, oL));
  if (om1 < m1) {
    m1 = om1;
    pb = opb;
    owner = oown;
  }
}

// The exact path's distance of key x to centroid c (the same fp32 operations
// in the same order as exact_assign).
__device__ __forceinline__ float exact_dist(const float (&x)[kRank], const float* mu, float nc2) {
  float dot = 0.f;
#pragma unroll
  for (int d = 0; d < kRank; ++d) dot = fmaf(x[d], mu[d], dot);
  return fmaf(-2.f, dot, nc2);
}

__global__ void __launch_bounds__(kMmaThreads, 3) km_assign_mma_kernel(const KmeansArgs a) {
  // dynamic: -2 mu as fp16 [ncp][16] (32 bytes per centroid, its two 16-byte
  // halves swapped when bit 2 of c is set, so that the eight rows of an
  // ldmatrix tile fall in distinct bank groups), then |mu|^2 [ncp] (fp32,
  // +inf for the padding centroids c >= nc)
  extern __shared__ __align__(16) uint8_t km_smem[];
  __shared__ float wmax[kMmaWarps];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int npairs = (a.nc + 15) / 16, ncp = 16 * npairs;
  uint8_t* mu16 = km_smem;
  float* nrm = reinterpret_cast<float*>(km_smem + static_cast<size_t>(ncp) * 32);
  const float* src = a.centroids + bk * a.nc * kRank;
  float mymax = 0.f;
  for (int c = tid; c < ncp; c += kMmaThreads) {
    float v[kRank];
    if (c < a.nc) {
      const float4* c4 = reinterpret_cast<const float4*>(src + static_cast<size_t>(c) * kRank);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 m = c4[w];
        v[4 * w] = m.x;
        v[4 * w + 1] = m.y;
        v[4 * w + 2] = m.z;
        v[4 * w + 3] = m.w;
      }
    } else {
#pragma unroll
      for (int d = 0; d < kRank; ++d) v[d] = 0.f;
    }
    float sq = 0.f;  // the exact path's |mu|^2: fma over the dims in order
#pragma unroll
    for (int d = 0; d < kRank; ++d) sq = fmaf(v[d], v[d], sq);
    nrm[c] = c < a.nc ? sq : INFINITY;
    if (c < a.nc) mymax = fmaxf(mymax, sq);  // (a NaN norm is caught below: M is then NaN)
    if (c < a.nc && !(sq <= INFINITY)) mymax = NAN;
    uint4* row = reinterpret_cast<uint4*>(mu16 + static_cast<size_t>(c) * 32);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float* q = v + 8 * h;
      row[h ^ ((c >> 2) & 1)] = make_uint4(half2_bits(-2.f * q[0], -2.f * q[1]), half2_bits(-2.f * q[2], -2.f * q[3]),
                                           half2_bits(-2.f * q[4], -2.f * q[5]), half2_bits(-2.f * q[6], -2.f * q[7]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, mymax, off);
    mymax = (mymax != mymax || o != o) ? NAN : fmaxf(mymax, o);
  }
  if (lane == 0) wmax[warp] = mymax;
  __syncthreads();
  float M2 = 0.f;
#pragma unroll
  for (int w = 0; w < kMmaWarps; ++w) M2 = (M2 != M2 || wmax[w] != wmax[w]) ? NAN : fmaxf(M2, wmax[w]);
  const float M = sqrtf(M2);
  const bool m_ok = M <= 8192.f;  // false for NaN

  const int g = lane >> 2, q4 = lane & 3;
  const uint32_t mu_base = static_cast<uint32_t>(__cvta_generic_to_shared(mu16));
  // ldmatrix row address of this lane: matrix lane/8 = (centroid half-tile
  // lane/16, dim half (lane/8)&1), row lane%8
  const int lrow = 8 * (lane >> 4) + (lane & 7), lhalf = (lane >> 3) & 1;
  const float* Xh = a.X + bk * a.n * kRank;
  for (int grp = 0; grp < kMmaGroups; ++grp) {
    const int base = blockIdx.x * kMmaKeysPerCta + (grp * kMmaWarps + warp) * 32;
    if (base >= a.n) break;  // (uniform over the warp)
    // A fragments: rows base + 16 mt + g (+8), dims 2q4, 2q4+1 and 2q4+8, 2q4+9
    uint32_t af[2][4];
    float xsq[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int j = min(base + 16 * mt + g + 8 * rr, a.n - 1);
        const float* xr = Xh + static_cast<size_t>(j) * kRank;
        const float2 lo = *reinterpret_cast<const float2*>(xr + 2 * q4);
        const float2 hi = *reinterpret_cast<const float2*>(xr + 2 * q4 + 8);
        af[mt][rr] = half2_bits(lo.x, lo.y);
        af[mt][2 + rr] = half2_bits(hi.x, hi.y);
        xsq[mt][rr] = fmaf(lo.x, lo.x, fmaf(lo.y, lo.y, fmaf(hi.x, hi.x, hi.y * hi.y)));
      }
    float m1[2][2], L[2][2];
    int pb[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        m1[mt][rr] = INFINITY;
        L[mt][rr] = INFINITY;
        pb[mt][rr] = 0;
      }
    for (int p = 0; p < npairs; ++p) {
      const int n0 = 16 * p;
      const int cr = n0 + lrow;
      uint32_t b00, b01, b10, b11;  // [centroid tile][dim half]
      ldsm_x4_b16(mu_base + cr * 32 + ((lhalf ^ ((cr >> 2) & 1)) << 4), b00, b01, b10, b11);
      const float2 c0 = *reinterpret_cast<const float2*>(nrm + n0 + 2 * q4);
      const float2 c1 = *reinterpret_cast<const float2*>(nrm + n0 + 8 + 2 * q4);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        float d0[4], d1[4];
        mma_f16(d0, af[mt], b00, b01, c0.x, c0.y);
        mma_f16(d1, af[mt], b10, b11, c1.x, c1.y);
        top2_group(m1[mt][0], L[mt][0], pb[mt][0], d0[0], d0[1], d1[0], d1[1], p);
        top2_group(m1[mt][1], L[mt][1], pb[mt][1], d0[2], d0[3], d1[2], d1[3], p);
      }
    }
    // the four threads of a quad saw different centroids of the same rows
    int own[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        own[mt][rr] = q4;
        top2_merge(m1[mt][rr], L[mt][rr], pb[mt][rr], own[mt][rr], 1);
        top2_merge(m1[mt][rr], L[mt][rr], pb[mt][rr], own[mt][rr], 2);
        xsq[mt][rr] += __shfl_xor_sync(0xffffffffu, xsq[mt][rr], 1);
        xsq[mt][rr] += __shfl_xor_sync(0xffffffffu, xsq[mt][rr], 2);
      }
    // lane (g, q4) decides row 16 (q4 >> 1) + g + 8 (q4 & 1) of the group
    const int mt = q4 >> 1, rr = q4 & 1;
    const float bm1 = mt ? (rr ? m1[1][1] : m1[1][0]) : (rr ? m1[0][1] : m1[0][0]);
    const float bm2 = mt ? (rr ? L[1][1] : L[1][0]) : (rr ? L[0][1] : L[0][0]);
    const int bpb = mt ? (rr ? pb[1][1] : pb[1][0]) : (rr ? pb[0][1] : pb[0][0]);
    const int bown = mt ? (rr ? own[1][1] : own[1][0]) : (rr ? own[0][1] : own[0][0]);
    const float bx2 = mt ? (rr ? xsq[1][1] : xsq[1][0]) : (rr ? xsq[0][1] : xsq[0][0]);
    const int j = base + 16 * mt + g + 8 * rr;
    const float xn = sqrtf(bx2);
    const float E = 0x1.2p-9f * xn * M + 0x1p-16f * M * M + 0x1p-20f * (xn + M);
    const bool sure = m_ok && xn < 30000.f && (bm2 - bm1) > 2.f * E;  // false for any NaN
    const bool valid = j < a.n;
    if (valid && sure) {
      // The nearest centroid is unique and is one of the four that the
      // owning lane saw in pair bpb (the one that gave m1): the smallest of
      // their exact distances (ascending order) is it.
      float xr[kRank];
      const float4* x4 = reinterpret_cast<const float4*>(Xh + static_cast<size_t>(j) * kRank);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 v = x4[w];
        xr[4 * w] = v.x;
        xr[4 * w + 1] = v.y;
        xr[4 * w + 2] = v.z;
        xr[4 * w + 3] = v.w;
      }
      float best = INFINITY;
      int bc = 16 * bpb + 2 * bown;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = 16 * bpb + 8 * (k >> 1) + 2 * bown + (k & 1);
        if (c < a.nc) {
          const float dist = exact_dist(xr, src + static_cast<size_t>(c) * kRank, nrm[c]);
          if (dist < best) {
            best = dist;
            bc = c;
          }
        }
      }
      a.assign[bk * a.n + j] = bc;
    }
    const uint32_t undecided = __ballot_sync(0xffffffffu, valid && !sure);
    if (undecided) {
      int slot0 = 0;
      if (lane == 0) slot0 = atomicAdd(a.amb_count + bk, __popc(undecided));
      slot0 = __shfl_sync(0xffffffffu, slot0, 0);
      if (valid && !sure) a.amb_list[bk * a.n + slot0 + __popc(undecided & ((1u << lane) - 1u))] = j;
    }
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

// Grouping of the keys by cluster, in four steps over many CTAs; the result
// is that of one walk over the keys in order: members of a cluster ascend,
// and each centroid is the sum of its members' projections in member order,
// divided by their number (an empty cluster keeps its centroid).
//   km_hist   per segment of kKmSegKeys keys: the count of each cluster
//   km_segscan per cluster: where each segment's keys start inside it, and
//             its size
//   km_scan   per (sequence, head): the offsets of the clusters
//   km_place  one warp per segment: its keys to their places, in key order
//   km_means  one half-warp per cluster: lane d sums dimension d
constexpr int kHistThreads = 256;
constexpr int kPlaceWarps = 4;
constexpr int kMeansThreads = 256;

__global__ void __launch_bounds__(kHistThreads) km_hist_kernel(const KmeansArgs a) {
  __shared__ int cnt[kMaxClusters];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int tid = threadIdx.x, sg = blockIdx.x;
  const int32_t* asg = a.assign + bk * a.n;
  for (int c = tid; c < a.nc; c += kHistThreads) cnt[c] = 0;
  __syncthreads();
  const int j1 = min(a.n, (sg + 1) * kKmSegKeys);
  for (int j = sg * kKmSegKeys + tid; j < j1; j += kHistThreads) atomicAdd(&cnt[asg[j]], 1);
  __syncthreads();
  int32_t* seg = a.seg + (bk * a.n_seg + sg) * a.nc;
  for (int c = tid; c < a.nc; c += kHistThreads) seg[c] = cnt[c];
}

// One thread per cluster: each segment's start relative to the cluster (in
// place over the counts) and the cluster's size (into its offsets entry).
constexpr int kSegScanThreads = 256;
__global__ void __launch_bounds__(kSegScanThreads) km_segscan_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int c = blockIdx.x * kSegScanThreads + threadIdx.x;
  if (c >= a.nc) return;
  int32_t* seg = a.seg + bk * a.n_seg * a.nc + c;
  int run = 0;
  for (int sg0 = 0; sg0 < a.n_seg; sg0 += 8) {  // eight segments' counts in flight, then their starts
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = sg0 + u < a.n_seg ? seg[static_cast<size_t>(sg0 + u) * a.nc] : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (sg0 + u < a.n_seg) {
        seg[static_cast<size_t>(sg0 + u) * a.nc] = run;
        run += v[u];
      }
  }
  a.offsets[bk * (a.nc + 1) + c] = run;
}

// One CTA per (sequence, head): the clusters' offsets from their sizes.
__global__ void __launch_bounds__(kGroupThreads) km_scan_kernel(const KmeansArgs a) {
  __shared__ int cnt[kMaxClusters], off[kMaxClusters];
  __shared__ int warp_tot[32];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int tid = threadIdx.x;
  if (tid == 0) a.amb_count[bk] = 0;  // the undecided list of the next round starts empty
  int32_t* offs = a.offsets + bk * (a.nc + 1);
  for (int c = tid; c < a.nc; c += kGroupThreads) cnt[c] = offs[c];
  __syncthreads();
  scan_counts(cnt, off, a.nc, warp_tot);
  __syncthreads();
  for (int c = tid; c < a.nc; c += kGroupThreads) offs[c] = off[c];
  if (tid == 0) offs[a.nc] = a.n;
}

__global__ void __launch_bounds__(32 * kPlaceWarps) km_place_kernel(const KmeansArgs a) {
  __shared__ int running[kPlaceWarps][kMaxClusters];
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int sg = blockIdx.x * kPlaceWarps + w;
  if (sg >= a.n_seg) return;  // (warp-uniform; the warps share no barrier)
  const int32_t* start = a.seg + (bk * a.n_seg + sg) * a.nc;  // relative to the cluster
  const int32_t* offs = a.offsets + bk * (a.nc + 1);
  for (int c = lane; c < a.nc; c += 32) running[w][c] = offs[c] + start[c];
  __syncwarp();
  const int32_t* asg = a.assign + bk * a.n;
  int32_t* mem = a.members + bk * a.n;
  const uint32_t lt = (1u << lane) - 1u;
  const int j1 = min(a.n, (sg + 1) * kKmSegKeys);
  for (int j0 = sg * kKmSegKeys; j0 < j1; j0 += 32 * 8) {
    int cj[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + 32 * u + lane;
      cj[u] = j < j1 ? asg[j] : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = cj[u];
      const uint32_t peers = __match_any_sync(0xffffffffu, c);
      if (c >= 0) mem[running[w][c] + __popc(peers & lt)] = a.block + j0 + 32 * u + lane;
      __syncwarp();
      if (c >= 0 && lane == __ffs(peers) - 1) running[w][c] += __popc(peers);
      __syncwarp();
    }
  }
}

__global__ void __launch_bounds__(kMeansThreads) km_means_kernel(const KmeansArgs a) {
  if (a.kind[blockIdx.y] != KIND_SPARSE) return;
  const size_t bk = head_index(a);
  const int c = (blockIdx.x * kMeansThreads + threadIdx.x) >> 4, d = threadIdx.x & 15;
  if (c >= a.nc) return;  // (no barriers or shuffles below)
  const int32_t* offs = a.offsets + bk * (a.nc + 1);
  const int o0 = offs[c], size = offs[c + 1] - o0;
  if (size == 0) return;
  const int32_t* mem = a.members + bk * a.n + o0;
  const float* Xd = a.X + bk * a.n * kRank + d;
  float s = 0.f;
  int e = 0;
  for (; e + 4 <= size; e += 4) {  // four members' loads in flight, added in order
    int jj[4];
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) jj[u] = mem[e + u] - a.block;
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = Xd[static_cast<size_t>(jj[u]) * kRank];
#pragma unroll
    for (int u = 0; u < 4; ++u) s += v[u];
  }
  for (; e < size; ++e) s += Xd[static_cast<size_t>(mem[e] - a.block) * kRank];
  a.centroids[(bk * a.nc + c) * kRank + d] = s / static_cast<float>(size);
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
  const size_t ncp = 16 * static_cast<size_t>((a.nc + 15) / 16);
  const size_t smem_mma = ncp * (32 + sizeof(float));
  // RTP_KMEANS_EXACT_ASSIGN=1 (diagnostic): every key by the exact fp32 path,
  // which the tensor-core pass must reproduce key for key.
  static const bool exact_only = [] {
    const char* e = std::getenv("RTP_KMEANS_EXACT_ASSIGN");
    return e && e[0] == '1';
  }();
  cudaError_t e = cudaFuncSetAttribute(km_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(km_rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(km_assign_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_mma));
  if (e != cudaSuccess) return e;
  const dim3 per_mma((a.n + kMmaKeysPerCta - 1) / kMmaKeysPerCta, a.n_kv_heads, a.batch);
  const dim3 per_seg(a.n_seg, a.n_kv_heads, a.batch);
  const dim3 per_segscan((a.nc + kSegScanThreads - 1) / kSegScanThreads, a.n_kv_heads, a.batch);
  const dim3 per_place((a.n_seg + kPlaceWarps - 1) / kPlaceWarps, a.n_kv_heads, a.batch);
  const dim3 per_means((a.nc * 16 + kMeansThreads - 1) / kMeansThreads, a.n_kv_heads, a.batch);
  // one CTA per chunk of a full list; those beyond the list's end leave at once
  const dim3 per_rescore = per_keys;
  for (int it = 0; it < iters; ++it) {
    if (exact_only) {
      km_assign_kernel<<<per_keys, kKmThreads, smem, stream>>>(a);
    } else {
      km_assign_mma_kernel<<<per_mma, kMmaThreads, smem_mma, stream>>>(a);
      km_rescore_kernel<<<per_rescore, kKmThreads, smem, stream>>>(a);
    }
    km_hist_kernel<<<per_seg, kHistThreads, 0, stream>>>(a);
    km_segscan_kernel<<<per_segscan, kSegScanThreads, 0, stream>>>(a);
    km_scan_kernel<<<per_head, kGroupThreads, 0, stream>>>(a);
    km_place_kernel<<<per_place, 32 * kPlaceWarps, 0, stream>>>(a);
    km_means_kernel<<<per_means, kMeansThreads, 0, stream>>>(a);
  }
  km_chunks_kernel<<<per_head, kGroupThreads, 0, stream>>>(a);
  if (a.k_sorted) {  // no cluster-ordered copy when the decode reads member rows in place
    const dim3 per_row((a.n + kKmThreads / 32 - 1) / (kKmThreads / 32), a.n_kv_heads, a.batch);
    km_permute_kernel<<<per_row, kKmThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace rtp
