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
  __shared__ float qsum[kHeadDim];
  __shared__ float part16[16][kRank];
  const int kvh = blockIdx.x, b = blockIdx.y;
  // The attention launch that follows may start now: its streaming-head
  // CTAs do not need the selection, its retrieval-head CTAs wait for it.
  griddep_launch_dependents();
  if (a.kind[kvh] != KIND_SPARSE) return;
  // qbar = sum_h P^T q_h = P^T (sum_h q_h): sum the group's queries (fixed
  // head order), then project with all threads: thread (j, c) takes dims
  // [8j, 8j+8) of output c, and the 16 partials are added in a fixed order.
  const int tid = threadIdx.x;
  if (tid < kHeadDim) {
    const __nv_bfloat16* qg = a.q + (static_cast<size_t>(b) * a.n_q_heads + kvh * a.group) * kHeadDim + tid;
    float sq = 0.f;
    for (int h = 0; h < a.group; ++h) sq += __bfloat162float(qg[h * kHeadDim]);
    qsum[tid] = sq;
  }
  __syncthreads();
  {
    const int j = tid >> 4, c = tid & 15;
    float sp = 0.f;
#pragma unroll
    for (int d = 8 * j; d < 8 * j + 8; ++d) sp = fmaf(__ldg(a.proj + d * kRank + c), qsum[d], sp);
    part16[j][c] = sp;
  }
  __syncthreads();
  float q[kRank];
#pragma unroll
  for (int c = 0; c < kRank; ++c) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) s += part16[j][c];
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

// --------------------------------------------------------------- attention
// One CTA per (span of <= 128 keys, KV head, sequence); 4 warps, warp w owns
// keys [32w, 32w+32) of the span.  K and V of the span arrive by TMA in
// 128-byte-swizzled 64x64 boxes (rows past the cache read as zero).  Per warp,
// tensor-core MMAs (m16n8k16, bf16 -> fp32) with the group's query heads as
// the 16 M rows (rows >= G are zero):
//   S = Q K^T   (A = Q fragments in registers, B = K via ldmatrix),
//   P = exp2(S * scale*log2e - m_warp) kept in registers as the A operand,
//   O = P V     (B = V via ldmatrix.trans).
// The four warps' (m, l, O) are merged in shared memory (reusing the K
// buffer) and the CTA writes one partial per head.
struct __align__(1024) DecSmem {
  uint8_t k[32768];  // 128 keys x 128 dims, two 64-column swizzled chunks
  uint8_t v[32768];
  uint64_t bar;
  float wm[4][16], wl[4][16];
  int ok;
};
constexpr size_t kDecSmemBytes = sizeof(DecSmem) + 1024;

__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int dim) {
  return base + (dim >> 6) * 16384 + row * 128 + ((((dim & 63) >> 3) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const __grid_constant__ CUtensorMap mk,
                                                                    const __grid_constant__ CUtensorMap mv,
                                                                    const DecodeArgs a) {
  extern __shared__ uint8_t dsmem[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int s = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.group;
  // Only retrieval heads read the selection written by the preceding launch.
  if (a.kind[kvh] == KIND_SPARSE) griddep_wait();
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
  const uint32_t ks = smem_u32(sm.k), vs = smem_u32(sm.v);
  const int slab = b * a.n_kv_heads + kvh;
  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&sm.bar, 65536);
    for (int cc = 0; cc < 2; ++cc)
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_3d(sm.k + cc * 16384 + hh * 8192, &mk, &sm.bar, 64 * cc, key0 + 64 * hh, slab);
        tma_load_3d(sm.v + cc * 16384 + hh * 8192, &mv, &sm.bar, 64 * cc, key0 + 64 * hh, slab);
      }
  }
  // Q as A fragments: rows g and g+8 are query heads g and g+8 of the group
  // (zero beyond G); 8 K steps of 16 dims.
  uint32_t qa[8][4];
  {
    const __nv_bfloat16* qb = a.q + (static_cast<size_t>(b) * a.n_q_heads + kvh * G) * kHeadDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d0 = 16 * kk + 2 * c;
      qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qb + g * kHeadDim + d0) : 0u;
      qa[kk][1] = g + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * kHeadDim + d0) : 0u;
      qa[kk][2] = g < G ? *reinterpret_cast<const uint32_t*>(qb + g * kHeadDim + d0 + 8) : 0u;
      qa[kk][3] = g + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * kHeadDim + d0 + 8) : 0u;
    }
  }
  if (tid == 0) sm.ok = mbar_wait(&sm.bar, 0, nullptr, a.status) ? 1 : 0;
  __syncwarp();
  __syncthreads();
  if (!sm.ok) return;

  // S = Q K^T over this warp's 32 keys: 4 n-tiles of 8 keys
  float sacc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
  const int kbase = 32 * warp;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      uint32_t r[4];
      const int key = kbase + 16 * np + (lane >> 4) * 8 + (lane & 7);
      const int dim = 16 * kk + ((lane >> 3) & 1) * 8;
      ldsm_x4(sw128(ks, key, dim), r);
      mma_bf16(sacc[2 * np], qa[kk], r[0], r[1]);
      mma_bf16(sacc[2 * np + 1], qa[kk], r[2], r[3]);
    }
  }
  // scale to log2 units, mask keys past the span, row maxima (rows g, g+8)
  const float sl2 = a.scale_log2;
  float mrow[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = kbase + 8 * n + 2 * c + (e & 1);
      const float v = key < nk ? sacc[n][e] * sl2 : -INFINITY;
      sacc[n][e] = v;
      mrow[e >> 1] = fmaxf(mrow[e >> 1], v);
    }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    mrow[rr] = fmaxf(mrow[rr], __shfl_xor_sync(0xffffffffu, mrow[rr], 1));
    mrow[rr] = fmaxf(mrow[rr], __shfl_xor_sync(0xffffffffu, mrow[rr], 2));
  }
  const float muse[2] = {mrow[0] == -INFINITY ? 0.f : mrow[0], mrow[1] == -INFINITY ? 0.f : mrow[1]};
  float lrow[2] = {0.f, 0.f};
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = exp2f(sacc[n][e] - muse[e >> 1]);
      sacc[n][e] = p;
      lrow[e >> 1] += p;
    }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 1);
    lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 2);
  }
  // O = P V: 16 n-tiles of 8 dims, 2 K steps of 16 keys
  float oacc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]);
    pa[1] = pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]);
    pa[2] = pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
    pa[3] = pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      uint32_t r[4];
      const int key = kbase + 16 * kk + ((lane >> 3) & 1) * 8 + (lane & 7);
      const int dim = 16 * dp + (lane >> 4) * 8;
      ldsm_x4_t(sw128(vs, key, dim), r);
      mma_bf16(oacc[2 * dp], pa, r[0], r[1]);
      mma_bf16(oacc[2 * dp + 1], pa, r[2], r[3]);
    }
  }
  // merge the four warps (K buffer reused as [warp][row][dim] fp32)
  __syncthreads();
  float (*wo)[16][128] = reinterpret_cast<float (*)[16][128]>(sm.k);
  if (c == 0) {
    sm.wm[warp][g] = mrow[0];
    sm.wm[warp][g + 8] = mrow[1];
    sm.wl[warp][g] = lrow[0];
    sm.wl[warp][g + 8] = lrow[1];
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    *reinterpret_cast<float2*>(&wo[warp][g][8 * n + 2 * c]) = make_float2(oacc[n][0], oacc[n][1]);
    *reinterpret_cast<float2*>(&wo[warp][g + 8][8 * n + 2 * c]) = make_float2(oacc[n][2], oacc[n][3]);
  }
  __syncthreads();
  const int d = tid;  // one output dimension per thread
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm.wm[w][h]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = sm.wm[w][h] == -INFINITY ? 0.f : exp2f(sm.wm[w][h] - M);
      L = fmaf(f, sm.wl[w][h], L);
      o = fmaf(f, wo[w][h][d], o);
    }
    part[h * kPartStride + 4 + d] = o;
    if (d == 0) {
      part[h * kPartStride + 0] = M;
      part[h * kPartStride + 1] = L;
    }
  }
}

// Log-sum-exp merge of the splits of one query head: the split statistics
// (m, l) are loaded in parallel and reduced in shared memory, then each
// thread streams one output dimension over the splits (independent,
// coalesced loads, four in flight).
__global__ void __launch_bounds__(kAttnThreads) decode_combine_kernel(const DecodeArgs a) {
  extern __shared__ float wsh[];  // [max_splits] split weights
  __shared__ float red[kAttnThreads / 32];
  __shared__ float Msh, Lsh;
  griddep_wait();  // partials of the preceding attention launch
  const int hq = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = hq / a.group, h = hq % a.group;
  const int kind = a.kind[kvh];
  int nsplit;
  if (kind == KIND_SPARSE) {
    nsplit = min(a.cnt[static_cast<size_t>(b) * a.n_kv_heads + kvh], a.kmax);
  } else {
    const int start = (kind == KIND_SWA) ? max(0, a.cache_len - a.window) : 0;
    nsplit = (a.cache_len - start + 127) / 128;
  }
  nsplit = max(0, min(nsplit, a.max_splits));
  const float* base = a.partial + (static_cast<size_t>(b) * a.n_kv_heads + kvh) * a.max_splits * a.group * kPartStride;
  // 1. M = max of the split maxima
  float m = -INFINITY;
  for (int sp = tid; sp < nsplit; sp += kAttnThreads) {
    const float v = base[(sp * a.group + h) * kPartStride];
    wsh[sp] = v;
    m = fmaxf(m, v);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (tid == 0) {
    float M = red[0];
    for (int w = 1; w < kAttnThreads / 32; ++w) M = fmaxf(M, red[w]);
    Msh = M;
  }
  __syncthreads();
  const float M = Msh;
  // 2. weights w_s = 2^(m_s - M) and L = sum w_s l_s
  float lsum = 0.f;
  for (int sp = tid; sp < nsplit; sp += kAttnThreads) {
    const float ms = wsh[sp];
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
    wsh[sp] = w;
    lsum = fmaf(w, base[(sp * a.group + h) * kPartStride + 1], lsum);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  __syncthreads();
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  if (tid == 0) {
    float L = 0.f;
    for (int w = 0; w < kAttnThreads / 32; ++w) L += red[w];
    Lsh = L;
  }
  __syncthreads();
  // 3. o_d = sum_s w_s o_s[d] / L
  const int d = tid;
  const float* od = base + h * kPartStride + 4 + d;
  const size_t stride = static_cast<size_t>(a.group) * kPartStride;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  int sp = 0;
  for (; sp + 3 < nsplit; sp += 4) {
    const float v0 = od[sp * stride], v1 = od[(sp + 1) * stride], v2 = od[(sp + 2) * stride], v3 = od[(sp + 3) * stride];
    acc0 = fmaf(wsh[sp], v0, acc0);
    acc1 = fmaf(wsh[sp + 1], v1, acc1);
    acc2 = fmaf(wsh[sp + 2], v2, acc2);
    acc3 = fmaf(wsh[sp + 3], v3, acc3);
  }
  for (; sp < nsplit; ++sp) acc0 = fmaf(wsh[sp], od[sp * stride], acc0);
  const float L = Lsh;
  const float out = L > 0.f ? ((acc0 + acc1) + (acc2 + acc3)) / L : 0.f;
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

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t stream) {
  const size_t sel_smem = static_cast<size_t>(a.nbc) * sizeof(uint32_t);
  if (sel_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
  }
  decode_select_kernel<<<dim3(a.n_kv_heads, a.batch), kSelThreads, sel_smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kDecSmemBytes));
  if (e != cudaSuccess) return e;
  // Programmatic dependent launches: each kernel may begin while the
  // previous one finishes; griddepcontrol.wait orders the data it reads.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.max_splits, a.n_kv_heads, a.batch);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = kDecSmemBytes;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_attn_kernel, mk, mv, a);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(a.n_q_heads, a.batch);
  cfg.dynamicSmemBytes = static_cast<size_t>(a.max_splits) * sizeof(float);
  if (cfg.dynamicSmemBytes > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(cfg.dynamicSmemBytes));
    if (e != cudaSuccess) return e;
  }
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel, a);
}

}  // namespace rtp
