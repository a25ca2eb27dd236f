// Sparse decode step: one new token per sequence over a KV cache.
//
// Page "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳": in the
// Qwen3-Coder experiment retrieval heads are sparsified in the decode phase
// while the streaming heads keep a window of 8192; the summary of "Full
// Attention Strikes Back" reports the decode speed-up.  For a retrieval head
// the query summary qbar = sum_{h in group} P^T q_h scores the cached block
// centroids, the sink + top-k + local blocks are selected (the prefill rule
// with t = the block of the new token), and exact softmax attention runs
// over the selected keys; streaming heads attend to the last `window` keys.
//
// Three launches on the caller's stream:
//  1. decode_select_kernel  (seq, retrieval head): summary + selection.
//  2. decode_attn_kernel    (split, kv head, seq): one span of <= 128 keys per
//     CTA.  K and V rows of the span are contiguous in the cache and are
//     brought into shared memory with two bulk copies on an mbarrier; QK runs
//     one key per thread, PV one output dimension per thread, for all G query
//     heads of the group at once (GQA: each K/V byte is read once per group).
//     Writes an unnormalised partial (m, l, o) per head in the log2 domain.
//  3. decode_combine_kernel (q head, seq): log-sum-exp merge of the splits.
// The step is bound by HBM reads of the selected K/V.

#include <cuda_bf16.h>

#include <mutex>

#include "internal.cuh"
#include "select_common.cuh"
#include "sm100.cuh"

namespace rtp {
namespace {

constexpr int kAttnThreads = 128;
constexpr int kMaxGroup = 16;

__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(const DecodeArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectScratch sh;
  __shared__ float proj_part[kMaxGroup][kRank];
  const int kvh = blockIdx.x, b = blockIdx.y;
  if (a.kind[kvh] != KIND_SPARSE) return;
  // per-head projections P^T q_h (fixed order over d), then the sum over heads
  const int tid = threadIdx.x;
  for (int e = tid; e < a.group * kRank; e += kSelThreads) {
    const int h = e / kRank, c = e % kRank;
    const __nv_bfloat16* qh = a.q + (static_cast<size_t>(b) * a.n_q_heads + kvh * a.group + h) * kHeadDim;
    float s = 0.f;
    for (int d = 0; d < kHeadDim; ++d) s = fmaf(a.proj[d * kRank + c], __bfloat162float(qh[d]), s);
    proj_part[h][c] = s;
  }
  __syncthreads();
  float q[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) {
    float s = 0.f;
    for (int h = 0; h < a.group; ++h) s += proj_part[h][c];
    q[c] = s;
  }
  const int t = (a.cache_len - 1) / a.block;
  const float* C = a.centroids + (static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.nbc * kRank;
  int32_t* out = a.sel + (static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.kmax;
  const int n = select_blocks(q, C, t, a.topk, a.n_local, a.kmax, keys, sh, out);
  if (tid == 0) a.cnt[static_cast<size_t>(b) * a.n_kv_heads + kvh] = n;
}

// Key span of split s for (b, kvh): [key0, key0 + nk).  nk <= 0: no work.
__device__ __forceinline__ void span_of(const DecodeArgs& a, int b, int kvh, int s, int& key0, int& nk) {
  const int kind = a.kind[kvh];
  if (kind == KIND_SPARSE) {
    const size_t bk = static_cast<size_t>(b) * a.n_kv_heads + kvh;
    const int cnt = a.cnt[bk];
    if (s >= cnt || s >= a.kmax) {
      nk = 0;
      key0 = 0;
      return;
    }
    int blk = a.sel[bk * a.kmax + s];
    const int t = (a.cache_len - 1) / a.block;
    if (blk < 0 || blk > t) {
      flag_error(a.status, RTP_DEVERR_INDEX);
      nk = 0;
      key0 = 0;
      return;
    }
    key0 = blk * a.block;
    nk = min(a.block, a.cache_len - key0);
  } else {
    const int start = (kind == KIND_SWA) ? max(0, a.cache_len - a.window) : 0;
    key0 = start + 128 * s;
    nk = min(128, a.cache_len - key0);
  }
}

// Dynamic shared memory: K span | V span (32 KB each) | q [G][128] fp32 |
// p [G][128] fp32.
size_t attn_smem_bytes(int group) { return 2 * 128 * kHeadDim * 2 + 2 * static_cast<size_t>(group) * 128 * 4; }

__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t dsmem[];
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(dsmem);
  __nv_bfloat16* vs = ks + 128 * kHeadDim;
  float* qs = reinterpret_cast<float*>(vs + 128 * kHeadDim);
  float (*ps)[128] = reinterpret_cast<float (*)[128]>(qs + a.group * kHeadDim);
  __shared__ float ms[kMaxGroup], ls[kMaxGroup];
  __shared__ uint64_t bar;
  __shared__ int ok_flag;
  const int s = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.group;
  float* part = a.partial + ((static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.max_splits + s) * G * kPartStride;
  int key0, nk;
  span_of(a, b, kvh, s, key0, nk);
  if (nk <= 0) {
    for (int h = 0; h < G; ++h) {
      if (tid == 0) {
        part[h * kPartStride + 0] = -INFINITY;
        part[h * kPartStride + 1] = 0.f;
      }
      part[h * kPartStride + 4 + tid] = 0.f;
    }
    return;
  }
  const size_t row0 = (static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.cache_len + key0;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint32_t bytes = static_cast<uint32_t>(nk) * kHeadDim * 2;
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_load(ks, a.kcache + row0 * kHeadDim, bytes, &bar);
    bulk_load(vs, a.vcache + row0 * kHeadDim, bytes, &bar);
  }
  // the group's queries, fp32
  for (int e = tid; e < G * kHeadDim; e += kAttnThreads) {
    const int h = e / kHeadDim, d = e % kHeadDim;
    qs[e] = __bfloat162float(a.q[(static_cast<size_t>(b) * a.n_q_heads + kvh * G + h) * kHeadDim + d]);
  }
  if (tid == 0) ok_flag = mbar_wait(&bar, 0, nullptr, a.status) ? 1 : 0;
  __syncwarp();  // warp 0 reconverges before the CTA barrier
  __syncthreads();
  if (!ok_flag) return;

  // QK: one key per thread; 16-byte chunks visited in a lane-rotated order
  // (keeps shared-memory bank conflicts at 2-way).
  {
    const int key = tid;
    float acc[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) acc[h] = 0.f;
    if (key < nk) {
      const uint4* krow = reinterpret_cast<const uint4*>(ks + key * kHeadDim);
      for (int c = 0; c < 16; ++c) {
        const int cc = (c + lane) & 15;
        const uint4 kv = krow[cc];
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(k2[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
          if (h < G) {
            const float4 q0 = *reinterpret_cast<const float4*>(&qs[h * kHeadDim + cc * 8]);
            const float4 q1 = *reinterpret_cast<const float4*>(&qs[h * kHeadDim + cc * 8 + 4]);
            float x = acc[h];
            x = fmaf(q0.x, kf[0], x);
            x = fmaf(q0.y, kf[1], x);
            x = fmaf(q0.z, kf[2], x);
            x = fmaf(q0.w, kf[3], x);
            x = fmaf(q1.x, kf[4], x);
            x = fmaf(q1.y, kf[5], x);
            x = fmaf(q1.z, kf[6], x);
            x = fmaf(q1.w, kf[7], x);
            acc[h] = x;
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < G) ps[h][key] = key < nk ? acc[h] * a.scale_log2 : -INFINITY;
  }
  __syncthreads();
  // softmax statistics per head (warp w handles heads w, w+4, ...)
  for (int h = warp; h < G; h += kAttnThreads / 32) {
    float m = -INFINITY;
    for (int x = lane; x < 128; x += 32) m = fmaxf(m, ps[h][x]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int x = lane; x < 128; x += 32) {
      const float p = exp2f(ps[h][x] - m);
      ps[h][x] = p;
      l += p;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      ms[h] = m;
      ls[h] = l;
    }
  }
  __syncthreads();
  // PV: one output dimension per thread, all heads
  {
    const int d = tid;
    float o[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) o[h] = 0.f;
    for (int x = 0; x < nk; ++x) {
      const float v = __bfloat162float(vs[x * kHeadDim + d]);
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h)
        if (h < G) o[h] = fmaf(ps[h][x], v, o[h]);
    }
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < G) part[h * kPartStride + 4 + d] = o[h];
    if (tid < G) {
      part[tid * kPartStride + 0] = ms[tid];
      part[tid * kPartStride + 1] = ls[tid];
    }
  }
}

__global__ void __launch_bounds__(kAttnThreads) decode_combine_kernel(const DecodeArgs a) {
  const int hq = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int kvh = hq / a.group, h = hq % a.group;
  const int kind = a.kind[kvh];
  int nsplit;
  if (kind == KIND_SPARSE) {
    nsplit = min(a.cnt[static_cast<size_t>(b) * a.n_kv_heads + kvh], a.kmax);
  } else {
    const int start = (kind == KIND_SWA) ? max(0, a.cache_len - a.window) : 0;
    nsplit = (a.cache_len - start + 127) / 128;
  }
  nsplit = min(nsplit, a.max_splits);
  const float* base = a.partial + (static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.max_splits * a.group * kPartStride;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, base[(s * a.group + h) * kPartStride]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* p = base + (s * a.group + h) * kPartStride;
    const float w = (p[0] == -INFINITY) ? 0.f : exp2f(p[0] - M);
    L = fmaf(w, p[1], L);
    acc = fmaf(w, p[4 + d], acc);
  }
  const float out = L > 0.f ? acc / L : 0.f;
  a.o[(static_cast<size_t>(b) * a.n_q_heads + hq) * kHeadDim + d] = __float2bfloat16_rn(out);
}

// Scratch of the allocation-free decode entry point: a file-scope device
// array that every GPU loading this library holds until the process exits.
static __device__ __align__(256) unsigned char g_decode_static_scratch[kDecodeStaticScratchBytes];

}  // namespace

cudaError_t decode_static_scratch(void** ptr) {
  // Host code may not use the array's name as a device address; look up the
  // address once per device, with that device current, and reuse it.
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const size_t sel_smem = static_cast<size_t>(a.nbc) * sizeof(uint32_t);
  if (sel_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
  }
  decode_select_kernel<<<dim3(a.n_kv_heads, a.batch), kSelThreads, sel_smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t attn_smem = attn_smem_bytes(a.group);
  e = cudaFuncSetAttribute(decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(attn_smem));
  if (e != cudaSuccess) return e;
  decode_attn_kernel<<<dim3(a.max_splits, a.n_kv_heads, a.batch), kAttnThreads, attn_smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(a.n_q_heads, a.batch), kAttnThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
