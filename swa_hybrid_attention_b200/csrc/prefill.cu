// Hybrid prefill attention (SWA / full causal / block-sparse heads) on the
// sm_100a tensor cores.
//
// What it computes: for query head h (KV head h / group) and query i,
//   O_i = softmax_j(scale * q_i . k_j) V   over the keys visible to the head:
//   SWA i-W < j <= i, full j <= i, sparse j <= i with block(j) selected for
//   i's query block.  (Pages: "阿里Qwen3 RTPurbo：15%全量Attention长文本5倍压缩方案"
//   — streaming heads drop far tokens, long-range heads keep full attention;
//   "阿里RTPurboV2：Transformer再次崛起，百步训练实现10倍稀少把稳" and the summary
//   of "Full Attention Strikes Back" — exact attention on the selected set.)
//
// Design (B200-first; the pages describe a Hopper kernel, not reused here):
//  * Persistent grid, one CTA per SM.  The work list (built on the host,
//    heaviest tiles first — the RTPurbo page's "sparsity-aware scheduling")
//    holds (KV head, pair of query heads of its group, 128-row query tile);
//    CTA c takes items c, c+grid, ...
//  * Both query heads of a pair visit the same KV tiles (same window, same
//    selection: the selection is shared by the group), so every K/V tile
//    loaded into shared memory feeds two S = Q K^T and two O += P V MMAs.
//    The four pairs of a group run on neighbouring CTAs at the same time,
//    so K/V are re-read from L2, not HBM.
//  * Warp roles: warp 0 = TMA producer (Q tiles, then a 2-stage K/V ring; a
//    stage's K is released as soon as both heads' S MMAs have read it and its
//    V after both P V MMAs, so the next K loads a tile earlier than V),
//    warp 1 = single-thread tcgen05.mma issuer, warp 2 = TMEM allocator,
//    warps 4-7 / 8-11 = softmax for head 0 / head 1 of the pair (one thread
//    per query row, the whole S row in registers: no cross-thread reduction).
//  * TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.  P (bf16)
//    is written back over the first 64 columns of its S and fed to the PV
//    MMA straight from TMEM (A operand in tensor memory).
//  * Online softmax in the log2 domain with a lazy reference maximum: O is
//    rescaled only when the row maximum grows by more than 2^8, so most
//    tiles never touch O from the CUDA cores.
//  * Masks are evaluated only on edge tiles (diagonal, window edge, sparse
//    diagonal); interior tiles run mask-free.
//  * Block size 64 (sparse heads): a 128-row query tile spans two query
//    blocks with different selections; the tile's KV list is the union of
//    both, loaded in 64-row halves, with a per-half membership mask.
//  * Every mbarrier wait is bounded; a time-out sets the device status word
//    and the CTA drains its in-flight copies/MMAs, frees TMEM and exits.

#include <cuda_bf16.h>

#include <climits>
#include <cstdint>

#include "exp2_poly.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace rtp {
namespace {

constexpr int kThreads = 384;
// Register split between roles (setmaxnreg): warpgroup 0 (producer, MMA,
// allocator, spare) gives registers to the two softmax warpgroups, which hold
// a whole 128-column S row each.  The split must fit in what the block is
// launched with (kThreads x kLaunchRegs), or the increase would wait forever;
// launch_prefill checks the compiled count.  The roles are separate
// (non-inlined) functions so that each is register-allocated for its own
// budget; each runs once per CTA.
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 88;
constexpr int kHighRegs = 200;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split must fit the launch");
// K/V rings of two stages each.  (A third K stage, loading K two tiles
// ahead, fits in shared memory but measured no faster on the 1M layer: the
// wait for K it removes moves to the P handshakes of the same chain.)
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128x128 bf16 operand tile
constexpr uint32_t kChunkBytes = 128 * 128;     // 64 columns x 128 rows
constexpr int kNoWindow = 1 << 30;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows > 2^8
constexpr uint32_t kMemberAll = 0x1Eu | (3u << 5);
// Column pairs (k mod 8) whose exponentials use the FMA-pipe polynomial
// instead of the MUFU: bit k set => pair k.  Default: none — measured on B200
// (1M-token layer) the polynomial costs more issue slots than the MUFU time
// it frees (1/8: +2.7 %, 1/4: +5.4 %, 3/8: +17 % kernel time).
#ifndef RTP_POLY_PAIRS
#define RTP_POLY_PAIRS 0x00u
#endif
constexpr uint32_t kPolyPairs = RTP_POLY_PAIRS;
// P is handed to the MMA issuer in kPChunks pieces of 128/kPChunks keys, so
// O += P V starts on the first keys while the softmax still exponentiates
// the rest (the P V of a tile then ends shortly after its softmax).
#ifndef RTP_P_CHUNKS
#define RTP_P_CHUNKS 2
#endif
constexpr int kPChunks = RTP_P_CHUNKS;
static_assert(kPChunks == 1 || kPChunks == 2 || kPChunks == 4, "P chunks must divide the four 32-key groups");

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kKStages], v_full[kVStages];
  uint64_t k_empty[kKStages];  // released once both heads' S MMAs of the tile have read K
  uint64_t v_empty[kVStages];  // released once both heads' P V MMAs have read V
  uint64_t s_full[2], o_full[2];
  uint64_t p_full[2][kPChunks];  // [head][chunk of keys]: that part of P is in TMEM
  uint64_t drain;
  uint32_t tile_mem[kKStages];  // per-head selections: the pair's membership of the tile in each K stage
  uint32_t tmem_base;
  int abort_flag;
};

struct Item {
  int kind, slot, b, kvh, bkv, pair, t;
};

__device__ __forceinline__ Item load_item(const int4* items, long idx, int n_kv_heads) {
  int4 w = items[idx];
  Item it;
  it.kind = w.x & 0xFF;
  it.slot = w.x >> 8;
  it.bkv = w.y;
  it.b = w.y / n_kv_heads;
  it.kvh = w.y - it.b * n_kv_heads;
  it.pair = w.z;
  it.t = w.w;
  return it;
}

// A KV tile: two 64-key halves starting at key positions row0 and row1.
// flags bit 0: the tile needs the element mask.  Bits 1..4: membership of
// (half 0, query half 0), (half 0, query half 1), (half 1, query half 0),
// (half 1, query half 1) — only block-64 sparse tiles clear any of them.
// Bits 5..6: membership of the pair's head 0 / head 1 — only per-head
// selections clear one of them (the tile is then the other head's).
struct TileRef {
  int row0, row1;
  uint32_t flags;
};

// Enumerates the KV tiles of one work item in ascending key order.  The
// producer, the MMA issuer and the softmax warps each run their own copy.
// kHeads: the selections are per query head (the pair's two lists are
// merged); a separate instantiation, so the shared-selection kernel carries
// none of its work.
template <bool kHeads>
struct TileIter {
  int kind, t, n, lo, q0, window, j;
  const int32_t* la;
  const int32_t* lb;
  int na, nb, ia, ib;
  int nblocks;  // valid block indices are < nblocks
  bool b64, heads;
  uint32_t* status;

  __device__ void init(const Item& it, const PrefillArgs& a) {
    kind = it.kind;
    t = it.t;
    j = 0;
    q0 = 128 * t;
    window = (kind == KIND_SWA) ? a.window : kNoWindow;
    b64 = false;
    heads = false;
    status = a.status;
    nblocks = a.nqb;
    if (kind == KIND_FULL) {
      lo = 0;
      n = t + 1;
    } else if (kind == KIND_SWA) {
      int first = q0 - a.window + 1;
      lo = first <= 0 ? 0 : first / 128;
      n = t - lo + 1;
    } else if (kHeads && a.block == 128) {
      // per-head selections: the union of the pair's two ascending lists
      heads = true;
      const long base = ((static_cast<long>(it.b) * a.n_sparse + it.slot) * a.group + 2 * it.pair) * a.nqb + t;
      la = a.sel + base * a.kmax;
      na = min(max(a.cnt[base], 0), a.kmax);
      lb = la + static_cast<long>(a.nqb) * a.kmax;
      nb = min(max(a.cnt[base + a.nqb], 0), a.kmax);
      int x = 0, y = 0, u = 0;
      while (x < na || y < nb) {
        int va = x < na ? la[x] : INT_MAX, vb = y < nb ? lb[y] : INT_MAX;
        if (va <= vb) ++x;
        if (vb <= va) ++y;
        ++u;
      }
      n = u;
      ia = ib = 0;
    } else if (a.block == 128) {
      long base = (static_cast<long>(it.b) * a.n_sparse + it.slot) * a.nqb + t;
      la = a.sel + base * a.kmax;
      na = min(max(a.cnt[base], 0), a.kmax);
      n = na;
    } else {
      b64 = true;
      long base = (static_cast<long>(it.b) * a.n_sparse + it.slot) * a.nqb + 2 * t;
      la = a.sel + base * a.kmax;
      na = min(max(a.cnt[base], 0), a.kmax);
      if (2 * t + 1 < a.nqb) {
        lb = la + a.kmax;
        nb = min(max(a.cnt[base + 1], 0), a.kmax);
      } else {
        lb = la;
        nb = 0;
      }
      // size of the union of the two ascending lists
      int x = 0, y = 0, u = 0;
      while (x < na || y < nb) {
        int va = x < na ? la[x] : INT_MAX, vb = y < nb ? lb[y] : INT_MAX;
        if (va <= vb) ++x;
        if (vb <= va) ++y;
        ++u;
      }
      n = (u + 1) / 2;
      ia = ib = 0;
    }
    if (n < 1) {
      // An empty selection cannot come from the selection kernel (the
      // diagonal block is always kept); treat it as the diagonal tile only.
      flag_error(status, RTP_DEVERR_INDEX);
      kind = KIND_FULL;
      window = kNoWindow;
      lo = t;
      n = 1;
    }
  }

  __device__ int checked_block(int blk, int limit) {
    if (blk < 0 || blk > limit) {
      flag_error(status, RTP_DEVERR_INDEX);
      return 0;
    }
    return blk;
  }

  // Next union entry (block-64 mode): value and membership (1 = A, 2 = B).
  __device__ bool pick(int& v, uint32_t& mem) {
    int va = ia < na ? la[ia] : INT_MAX, vb = ib < nb ? lb[ib] : INT_MAX;
    if (va == INT_MAX && vb == INT_MAX) return false;
    v = min(va, vb);
    mem = (va == v ? 1u : 0u) | (vb == v ? 2u : 0u);
    if (va == v) ++ia;
    if (vb == v) ++ib;
    return true;
  }

  __device__ TileRef next() {
    TileRef r;
    if (kind == KIND_FULL || kind == KIND_SWA) {
      int k0 = 128 * (lo + j);
      r.row0 = k0;
      r.row1 = k0 + 64;
      bool full_visible = (k0 + 127 <= q0) && (k0 > q0 + 127 - window);
      r.flags = kMemberAll | (full_visible ? 0u : 1u);
    } else if (kHeads && heads) {
      int v = 0;
      uint32_t m = 0;
      pick(v, m);
      const int blk = checked_block(v, t);
      r.row0 = 128 * blk;
      r.row1 = r.row0 + 64;
      // a head outside the tile's lists skips it whole (P = 0); the element
      // mask is only needed on the diagonal, which both lists hold
      r.flags = 0x1Eu | (m << 5) | (blk >= t ? 1u : 0u);
    } else if (!b64) {
      int blk = checked_block(la[j], t);
      r.row0 = 128 * blk;
      r.row1 = r.row0 + 64;
      r.flags = kMemberAll | (blk >= t ? 1u : 0u);
    } else {
      int v0 = 0, v1 = 0;
      uint32_t m0 = 0, m1 = 0;
      pick(v0, m0);
      if (!pick(v1, m1)) {
        v1 = v0;
        m1 = 0;
      }
      v0 = checked_block(v0, 2 * t + 1);
      v1 = checked_block(v1, 2 * t + 1);
      r.row0 = 64 * v0;
      r.row1 = 64 * v1;
      r.flags = 1u | ((m0 & 1u) << 1) | ((m0 & 2u) << 1) | ((m1 & 1u) << 3) | ((m1 & 2u) << 3) | (3u << 5);
    }
    ++j;
    return r;
  }
};

// Bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  return mbar_wait(bar, parity, nullptr, status);
}

// One lane polls, the whole warp gets the (uniform) result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  int ok = 1;
  if (lane_id() == 0) ok = mbar_wait(bar, parity, abort, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// ------------------------------------------------------------------ producer
template <bool kHeads>
__device__ __noinline__ void run_producer(Smem& s, const CUtensorMap* mq, const CUtensorMap* mk, const CUtensorMap* mv,
                             const PrefillArgs& a, volatile int* abort) {
  uint32_t it = 0, gt = 0;
  uint32_t k_issued = 0, v_issued = 0;  // K / V tiles whose copies were issued
  uint32_t q_issued = 0;  // bit h: Q of head h issued for the current item
  for (long idx = blockIdx.x; idx < a.n_items; idx += gridDim.x, ++it) {
    Item item = load_item(a.items, idx, a.n_kv_heads);
    const int zq = item.b * a.n_q_heads + item.kvh * a.group + 2 * item.pair;
    q_issued = 0;
    for (int h = 0; h < 2; ++h) {
      if (!mbar_wait(&s.q_empty[h], (it & 1u) ^ 1u, abort, a.status)) goto drain;
      mbar_arrive_expect_tx(&s.q_full[h], kTileBytes);
      tma_load_3d(s.q[h], mq, &s.q_full[h], 0, 128 * item.t - a.q_row0, zq + h);
      tma_load_3d(s.q[h] + kChunkBytes, mq, &s.q_full[h], 64, 128 * item.t - a.q_row0, zq + h);
      q_issued |= 1u << h;
    }
    {
      TileIter<kHeads> ti;
      ti.init(item, a);
      for (int j = 0; j < ti.n; ++j, ++gt) {
        TileRef tr = ti.next();
        const int sk = static_cast<int>(gt % kKStages), sv = static_cast<int>(gt % kVStages);
        const uint32_t uk = gt / kKStages, uv = gt / kVStages;
        if (!mbar_wait(&s.k_empty[sk], (uk & 1u) ^ 1u, abort, a.status)) goto drain;
        if constexpr (kHeads) s.tile_mem[sk] = (tr.flags >> 5) & 3u;  // published by the arrive below
        mbar_arrive_expect_tx(&s.k_full[sk], kTileBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(s.k[sk] + c * kChunkBytes, mk, &s.k_full[sk], 64 * c, tr.row0, item.bkv);
          tma_load_3d(s.k[sk] + c * kChunkBytes + kChunkBytes / 2, mk, &s.k_full[sk], 64 * c, tr.row1, item.bkv);
        }
        ++k_issued;
        if (!mbar_wait(&s.v_empty[sv], (uv & 1u) ^ 1u, abort, a.status)) goto drain;
        mbar_arrive_expect_tx(&s.v_full[sv], kTileBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(s.v[sv] + c * kChunkBytes, mv, &s.v_full[sv], 64 * c, tr.row0, item.bkv);
          tma_load_3d(s.v[sv] + c * kChunkBytes + kChunkBytes / 2, mv, &s.v_full[sv], 64 * c, tr.row1, item.bkv);
        }
        ++v_issued;
      }
    }
  }
  return;
drain:
  // Give up: wait (bounded) for the copies already issued so that no TMA
  // write lands in shared memory after the CTA has exited.
  for (uint32_t x = 0; x < kKStages && x < k_issued; ++x) {
    const uint32_t g = k_issued - 1 - x;
    drain_wait(&s.k_full[g % kKStages], (g / kKStages) & 1u, a.status);
  }
  for (uint32_t x = 0; x < kVStages && x < v_issued; ++x) {
    const uint32_t g = v_issued - 1 - x;
    drain_wait(&s.v_full[g % kVStages], (g / kVStages) & 1u, a.status);
  }
  for (int h = 0; h < 2; ++h)
    if (q_issued & (1u << h)) drain_wait(&s.q_full[h], it & 1u, a.status);
}

// ---------------------------------------------------------------- MMA issue
// The MMA thread's waits: a non-blocking test first (most phases it waits for
// have completed already, and the suspending try_wait costs ~150 cycles even
// then; this thread is the serial link between the softmax warps and the
// tensor pipe, so its own latencies add up), the bounded suspending wait
// otherwise.
__device__ __forceinline__ bool mbar_test_nb(uint64_t* bar, uint32_t parity) {  // test_wait: never suspends
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mma_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  if (mbar_test_nb(bar, parity)) return true;
  return mbar_wait(bar, parity, abort, status);
}
// The single issuing thread shares its scheduler with two busy softmax warps
// and the tensor pipe buffers very few MMAs, so the issue path is kept short:
// operand descriptors are built once per kernel and an operand at base + off
// is the base descriptor plus off >> 4 (the 14-bit start-address field counts
// 16-byte units; every shared address here is below 256 KB, so it never
// carries).  Stages and heads are picked with selects, not runtime-indexed
// arrays, which would live in local memory.
__device__ __forceinline__ constexpr uint64_t desc_off(uint32_t off_bytes) { return off_bytes >> 4; }

// S = Q K^T: M=128, N=128, K=128 (8 steps of 16); both operands K-major SW128.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t qd, uint64_t kd, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t off = desc_off((kk >> 2) * kChunkBytes + (kk & 3) * 32);
    umma_ss(d_tmem, qd + off, kd + off, idesc, kk > 0 ? 1u : 0u);
  }
}
// O += P V for key steps [kk0, kk1): P (bf16) from TMEM; V MN-major (16 keys
// = 2048 bytes per K-step, the two 64-dim chunks kChunkBytes apart).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t vd, uint32_t idesc,
                                         bool accumulate, int kk0, int kk1) {
#pragma unroll
  for (int kk = kk0; kk < kk1; ++kk)
    umma_ts(d_tmem, p_tmem + kk * 8, vd + desc_off(kk * 2048), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// O += P V of one head, each chunk of keys issued as soon as its part of P is
// in TMEM.  Returns false if a wait gave up.
__device__ __forceinline__ bool issue_pv_chunked(Smem& s, int h, uint32_t parity, uint32_t d_tmem, uint32_t p_tmem,
                                                 uint64_t vd, uint32_t idesc, bool accumulate, volatile int* abort,
                                                 uint32_t* status) {
#pragma unroll
  for (int q = 0; q < kPChunks; ++q) {
    // a polling loop here would take issue slots from the two softmax warps
    // that share this scheduler (measured ~1 % slower than suspending)
    if (!mma_wait(&s.p_full[h][q], parity, abort, status)) return false;
    tc_fence_after();
    issue_pv(d_tmem, p_tmem, vd, idesc, accumulate, q * (8 / kPChunks), (q + 1) * (8 / kPChunks));
  }
  return true;
}

// Head h's O += P V for the tile or, for a head outside the tile's lists
// (per-head selections), only the wait for its P handshake.
template <bool kHeads>
__device__ __forceinline__ bool pv_or_skip(Smem& s, int h, bool member, uint32_t parity, uint32_t d_tmem,
                                          uint32_t p_tmem, uint64_t vd, uint32_t idesc, bool accumulate,
                                          volatile int* abort, uint32_t* status) {
  if constexpr (kHeads) {
    if (!member) {
#pragma unroll
      for (int q = 0; q < kPChunks; ++q)
        if (!mma_wait(&s.p_full[h][q], parity, abort, status)) return false;
      return true;
    }
  }
  return issue_pv_chunked(s, h, parity, d_tmem, p_tmem, vd, idesc, accumulate, abort, status);
}

template <bool kHeads>
__device__ __noinline__ void run_mma(Smem& s, uint32_t tmem, const PrefillArgs& a, volatile int* abort) {
  const uint32_t id_qk = idesc_bf16_f32(128, 128, false);
  const uint32_t id_pv = idesc_bf16_f32(128, 128, true);
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 384};
  const uint64_t qd0 = smem_desc_sw128(smem_u32(s.q[0]), 16, 1024), qd1 = smem_desc_sw128(smem_u32(s.q[1]), 16, 1024);
  const uint64_t kd0 = smem_desc_sw128(smem_u32(s.k[0]), 16, 1024), kd1 = smem_desc_sw128(smem_u32(s.k[1]), 16, 1024);
  const uint64_t vd0 = smem_desc_sw128(smem_u32(s.v[0]), kChunkBytes, 1024);
  const uint64_t vd1 = smem_desc_sw128(smem_u32(s.v[1]), kChunkBytes, 1024);
  uint32_t it = 0, gt = 0, pc = 0;
  for (long idx = blockIdx.x; idx < a.n_items; idx += gridDim.x, ++it) {
    Item item = load_item(a.items, idx, a.n_kv_heads);
    TileIter<kHeads> ti;
    ti.init(item, a);
    const int n = ti.n;
    if (!mma_wait(&s.q_full[0], it & 1u, abort, a.status)) goto drain;
    if (!mma_wait(&s.q_full[1], it & 1u, abort, a.status)) goto drain;
    // per-head selections: membership of the tile in flight; a head's S and
    // P V are issued only for its own tiles (its s_full is still committed,
    // so the handshakes keep their phases), and its first P V overwrites O
    uint32_t mem_cur = 3u;
    bool started0 = false, started1 = false;
    {
      const int st0 = static_cast<int>(gt % kKStages);
      if (!mma_wait(&s.k_full[st0], (gt / kKStages) & 1u, abort, a.status)) goto drain;
      tc_fence_after();
      if constexpr (kHeads) mem_cur = s.tile_mem[st0];
      const uint64_t sk = st0 ? kd1 : kd0;
      if (!kHeads || (mem_cur & 1u)) issue_qk(tS[0], qd0, sk, id_qk);
      umma_commit(&s.s_full[0]);
      if (!kHeads || (mem_cur & 2u)) issue_qk(tS[1], qd1, sk, id_qk);
      umma_commit(&s.s_full[1]);
      umma_commit(&s.k_empty[st0]);
      if (n == 1) {
        umma_commit(&s.q_empty[0]);
        umma_commit(&s.q_empty[1]);
      }
    }
    for (int j = 0; j < n; ++j) {
      const uint32_t g = gt + j;
      const int st = static_cast<int>(g % kVStages);
      const bool has_next = j + 1 < n;
      const int st2 = static_cast<int>((g + 1) % kKStages);
      const uint64_t sv = st ? vd1 : vd0;
      const uint64_t sk2 = st2 ? kd1 : kd0;
      if (!mma_wait(&s.v_full[st], (g / kVStages) & 1u, abort, a.status)) goto drain;
      uint32_t mem_next = 3u;
      // head 0: O0 += P0 V ; then S0 for the next tile
      if (!pv_or_skip<kHeads>(s, 0, (mem_cur & 1u) != 0, pc & 1u, tO[0], tS[0], sv, id_pv, kHeads ? started0 : j > 0,
                              abort, a.status))
        goto drain;
      if (kHeads && (mem_cur & 1u)) started0 = true;
      if (!has_next) {
        umma_commit(&s.o_full[0]);
      } else {
        if (!mma_wait(&s.k_full[st2], ((g + 1) / kKStages) & 1u, abort, a.status)) goto drain;
        tc_fence_after();
        if constexpr (kHeads) mem_next = s.tile_mem[st2];
        if (!kHeads || (mem_next & 1u)) issue_qk(tS[0], qd0, sk2, id_qk);
        umma_commit(&s.s_full[0]);
        if (j + 2 == n) umma_commit(&s.q_empty[0]);
      }
      // head 1
      if (!pv_or_skip<kHeads>(s, 1, (mem_cur & 2u) != 0, pc & 1u, tO[1], tS[1], sv, id_pv, kHeads ? started1 : j > 0,
                              abort, a.status))
        goto drain;
      if (kHeads && (mem_cur & 2u)) started1 = true;
      umma_commit(&s.v_empty[st]);
      if (!has_next) {
        umma_commit(&s.o_full[1]);
      } else {
        if (!kHeads || (mem_next & 2u)) issue_qk(tS[1], qd1, sk2, id_qk);
        umma_commit(&s.s_full[1]);
        umma_commit(&s.k_empty[st2]);
        if (j + 2 == n) umma_commit(&s.q_empty[1]);
      }
      mem_cur = mem_next;
      ++pc;
    }
    gt += n;
  }
drain:
  // All MMAs issued by this thread must finish before TMEM is released.
  umma_commit(&s.drain);
  drain_wait(&s.drain, 0, a.status);
}

// ------------------------------------------------------------------ softmax
template <bool kHeads>
__device__ __noinline__ void run_softmax(Smem& s, uint32_t tmem, int h, const PrefillArgs& a, volatile int* abort) {
  const int q4 = warp_id() & 3;
  const int row = q4 * 32 + lane_id();
  const uint32_t lane_bits = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t tS = tmem + 128 * h + lane_bits;
  const uint32_t tO = tmem + 256 + 128 * h + lane_bits;
  const float sl2 = a.scale_log2;
  uint32_t it = 0, sc = 0;
  for (long idx = blockIdx.x; idx < a.n_items; idx += gridDim.x, ++it) {
    Item item = load_item(a.items, idx, a.n_kv_heads);
    TileIter<kHeads> ti;
    ti.init(item, a);
    const int i = 128 * item.t + row;
    const int rh = row >> 6;
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < ti.n; ++j) {
      const TileRef tr = ti.next();
      if (!warp_wait(&s.s_full[h], sc & 1u, abort, a.status)) return;
      ++sc;
      tc_fence_after();
      if (kHeads && !((tr.flags >> (5 + h)) & 1u)) {
        // a tile of the other head's list only: no S was computed for this
        // head and no P V will read its P; the handshake keeps the phases
#pragma unroll
        for (int q = 0; q < kPChunks; ++q) mbar_arrive(&s.p_full[h][q]);
        continue;
      }
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_ld_wait();
      if (tr.flags & 1u) {
        const int lo_key = i - ti.window;  // visible iff lo_key < key <= i
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int half = c >> 6;
          const int key = (half ? tr.row1 : tr.row0) + (c & 63);
          const bool member = kHeads ? (((tr.flags >> (1 + 2 * half + rh)) & (tr.flags >> (5 + h))) & 1u) != 0
                                     : ((tr.flags >> (1 + 2 * half + rh)) & 1u) != 0;
          if (!(member && key <= i && key > lo_key)) r[c] = __float_as_uint(-INFINITY);
        }
      }
      // row maximum: three-input max, four independent chains
      float m4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) m4[e] = max3(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]), -INFINITY);
#pragma unroll
      for (int k = 4; k < 64; ++k) m4[k & 3] = max3(m4[k & 3], __uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
      const float mx = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      const float m_new = mx * sl2;
      // Lazy rescale: a row moves its reference maximum only when the new
      // maximum exceeds it by more than 2^8.  O lives in TMEM and the
      // tcgen05.ld/st that rescale it are warp-collective, so the whole warp
      // takes the rescale path when any of its rows needs it (alpha = 1 for
      // the others).
      const bool raise = m_new > m_ref + kRescaleThreshold;
      const bool rescale_o = raise && j > 0 && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, rescale_o)) {
        const float alpha = rescale_o ? exp2f(m_ref - m_new) : 1.0f;
        l *= alpha;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
        tmem_st_wait();
      }
      if (raise) m_ref = m_new;
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      // P = exp2(s * scale*log2e - m) as packed bf16 pairs, written over the
      // first 64 columns of S (the whole S row is already in registers).
      // Arithmetic runs on packed f32x2 pairs; the column pairs selected by
      // kPolyPairs use the FMA-pipe polynomial, the others the MUFU ex2 (at
      // full tensor rate the MUFU alone could not keep up).
      const uint64_t sl2x2 = pack2(sl2, sl2), negm2 = pack2(-m_use, -m_use);
      uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t p[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int k = 16 * c + e;  // column pair (2k, 2k+1)
          const uint64_t x = fma2((static_cast<uint64_t>(r[2 * k + 1]) << 32) | r[2 * k], sl2x2, negm2);
          uint64_t pe;
          if ((kPolyPairs >> (k & 7)) & 1u)
            pe = exp2_poly2(lo2(x), hi2(x));
          else
            pe = pack2(exp2f(lo2(x)), exp2f(hi2(x)));
          s4[k & 3] = add2(s4[k & 3], pe);
          p[e] = pack_bf16x2(lo2(pe), hi2(pe));
        }
        tmem_st16(tS + 16 * c, p);
        if ((c + 1) % (4 / kPChunks) == 0) {  // a chunk of P is complete
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&s.p_full[h][c / (4 / kPChunks)]);
        }
      }
      {
        const uint64_t sa = add2(add2(s4[0], s4[1]), add2(s4[2], s4[3]));
        l += lo2(sa) + hi2(sa);
      }
    }
    // epilogue: O / l -> bf16
    if (!warp_wait(&s.o_full[h], it & 1u, abort, a.status)) return;
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int hq = item.kvh * a.group + 2 * item.pair + h;
    __nv_bfloat16* orow =
        a.o + ((static_cast<size_t>(item.b) * a.n_q_heads + hq) * static_cast<size_t>(a.q_slab) + (i - a.q_row0)) *
                  kHeadDim;
    const bool valid = i - a.q_row0 < a.q_rows;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
    tc_fence_before();
  }
}

template <bool kHeads>
__global__ void __launch_bounds__(kThreads, 1)
    hybrid_prefill_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                          const __grid_constant__ CUtensorMap mv, const __grid_constant__ PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = warp_id();
  if (threadIdx.x == 0) {
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s.q_full[h], 1);
      mbar_init(&s.q_empty[h], 1);
      mbar_init(&s.s_full[h], 1);
      for (int q = 0; q < kPChunks; ++q) mbar_init(&s.p_full[h][q], 128);
      mbar_init(&s.o_full[h], 1);
    }
    for (int st = 0; st < kKStages; ++st) {
      mbar_init(&s.k_full[st], 1);
      mbar_init(&s.k_empty[st], 1);
    }
    for (int st = 0; st < kVStages; ++st) {
      mbar_init(&s.v_full[st], 1);
      mbar_init(&s.v_empty[st], 1);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane_id() == 0) {
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
  }
  __syncwarp();
  if (warp == 2) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort = &s.abort_flag;

  // Each setmaxnreg sits inside its role's branch so that the raised budget
  // dominates only the softmax code.  Single-lane roles: the other 31 lanes
  // of warps 0 and 1 wait at __syncwarp so that every warp reaches the CTA
  // barrier below converged.
  if (warp >= 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    run_softmax<kHeads>(s, tmem, (warp - 4) >> 2, a, abort);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0) {
      if (lane_id() == 0) run_producer<kHeads>(s, &mq, &mk, &mv, a, abort);
      __syncwarp();
    } else if (warp == 1) {
      if (lane_id() == 0) run_mma<kHeads>(s, tmem, a, abort);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t prefill_smem_bytes() { return sizeof(Smem) + 1024; }

namespace {
template <bool kHeads>
cudaError_t launch_prefill_t(const PrefillArgs& a, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, int num_ctas, cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    // The setmaxnreg split is only valid for the register count it was sized
    // for; refuse to launch a build that compiled to anything else.
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, hybrid_prefill_kernel<kHeads>);
    if (e != cudaSuccess) return e;
    if (attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(hybrid_prefill_kernel<kHeads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(prefill_smem_bytes()));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  hybrid_prefill_kernel<kHeads><<<num_ctas, kThreads, prefill_smem_bytes(), stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           int num_ctas, cudaStream_t stream) {
  return a.sel_heads ? launch_prefill_t<true>(a, mq, mk, mv, num_ctas, stream)
                     : launch_prefill_t<false>(a, mq, mk, mv, num_ctas, stream);
}

}  // namespace rtp
