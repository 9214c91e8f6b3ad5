// Backward pass of the fused attention for B200 (sm_100a): dQ, dK, dV.
//
// The score matrix is not stored by the forward pass; it is recomputed here
// from Q, K and the forward's logsumexp ("理解 Flash Attention", section
// "瓦片注意力计算": S is needed for backpropagation and recomputed there, which
// keeps memory O(n)).  With P_ij = exp(scale q_i.k_j - lse_i) over visible keys:
//   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Two launches of one kernel template, no atomics:
//  * kDQ = true, stationary on a 128-row query tile (Q, dO copied into tensor
//    memory by the elementwise warpgroups, as the A operands): per visible
//    key tile j, S = Q K_j^T and dP = dO V_j^T, then the elementwise dS (one
//    thread per query row, bf16 written over S), then dQ += dS K_j.  It also
//    writes D_i to the workspace for the second launch.
//  * kDQ = false, stationary on a 128-key tile (K, V): per query tile i that
//    sees it, S^T = K Q_i^T and dP^T = V dO_i^T, the elementwise P^T and dS^T
//    (one thread per key row), then dV += P^T dO_i and dK += dS^T Q_i.
//
// Warp roles (384 threads, one CTA per SM): warp 0 issues the MMAs, warp 1
// is the TMA producer, warps 4-7 and 8-11 are two elementwise warpgroups.
// Every streamed tile is processed in two halves of 64 columns (keys for
// kDQ, queries otherwise); warpgroup h owns half h.  The halves have their
// own tensor-memory buffers, so while one warpgroup works on its half the
// tensor core computes the other half's scores or the accumulation of the
// half just finished:
//   S_0 dP_0 | S_1 dP_1 | (wait P_0) acc_0, S_0' dP_0' | (wait P_1) acc_1, S_1' dP_1' | ...
// Every barrier wait is bounded as in the forward kernel; on expiry the CTA
// records FA_ERR_DEVICE_TIMEOUT, leaves its loops, drains and frees TMEM.
#pragma once

#include <type_traits>

#include "fa_fwd_kernel.cuh"

namespace fa {

struct BwdParams {
  CUtensorMap tm_q;   // [B*H][Nq][D] bf16, box 64 x 128 x 1, 128B swizzle
  CUtensorMap tm_k;   // [B*H][Nk][D]
  CUtensorMap tm_v;   // [B*H][Nk][D]
  CUtensorMap tm_do;  // [B*H][Nq][D]
  const __nv_bfloat16* q;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;  // [B*H][Nq]
  float* delta;      // [B*H][Nq], written by the kDQ launch
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const uint8_t* mask;  // nullptr or [B*H][nqt][nkt]
  int Nq, Nk, nqt, nkt, causal_off, bh, causal;
  float scale, scale_log2;
  unsigned long long timeout_ns;
  int* status;
};

constexpr int kBwdThreads = 384;
constexpr int kBwdMmaWarp = 0;
constexpr int kBwdLoadWarp = 1;
constexpr int kBwdFirstEwWarp = 4;  // warps 4-7: half 0, warps 8-11: half 1

template <int D>
struct BwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages = (D == 128) ? 2 : 4;  // streamed tile pairs in flight
  // Shared memory: stationary tiles A, B (kDQ: Q, dO; else K, V), the ring of
  // streamed pairs X, Y (kDQ: K_j, V_j; else Q_i, dO_i), and for the dK/dV
  // launch the column values of each ring slot (-log2(e) lse_q, -D_q).
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kTileBytes;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffVals = kOffRing + kStages * 2 * kTileBytes;
  static constexpr int kOffBar = kOffVals + kStages * 2 * 128 * 4;
  // ab_full, ab_empty, full[S], empty[S], s_full[2], p_full[2], acc_full,
  // acc_empty, mma_done
  static constexpr int kNumBars = 2 + 2 * kStages + 4 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  // Tensor memory: half h has scores at [128h, 128h + 64) and their gradient
  // (dP or dP^T) at [128h + 64, 128h + 128); the bf16 results are written
  // over the first 32 columns of each.  Accumulators: kDQ: dQ at [256, 256 + D);
  // else dV at [256, 256 + D) and dK at [256 + D, 256 + 2D).
  // The dQ launch also keeps Q and dO in tensor memory ([256 + D, 256 + 3D/2)
  // and [256 + 3D/2, 256 + 2D), bf16 pairs per column) as the A operands of S
  // and dP: then the 64-wide score MMAs read only K and V from shared memory.
  static constexpr uint32_t kAcc0 = 256;
  static constexpr uint32_t kAcc1 = 256 + D;
  static constexpr uint32_t kTq = 256 + D;
  static constexpr uint32_t kTdo = 256 + D + D / 2;
  __host__ __device__ static constexpr uint32_t s_col(int h) { return 128u * h; }
  __host__ __device__ static constexpr uint32_t g_col(int h) { return 128u * h + 64u; }
};

struct BwdBars {
  uint32_t b0;
  int stages;
  __device__ uint32_t ab_full() const { return b0; }
  __device__ uint32_t ab_empty() const { return b0 + 8; }
  __device__ uint32_t full(int s) const { return b0 + 16 + 8u * s; }
  __device__ uint32_t empty(int s) const { return b0 + 16 + 8u * (stages + s); }
  __device__ uint32_t s_full(int h) const { return b0 + 16 + 16u * stages + 8u * h; }
  __device__ uint32_t p_full(int h) const { return b0 + 32 + 16u * stages + 8u * h; }
  __device__ uint32_t acc_full() const { return b0 + 48 + 16u * stages; }
  __device__ uint32_t acc_empty() const { return b0 + 56 + 16u * stages; }
  __device__ uint32_t mma_done() const { return b0 + 64 + 16u * stages; }
};

// Bounded wait by one thread; false on time-out or (honor_abort) abort.
__device__ __forceinline__ bool bwd_wait1(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          const BwdParams& p, bool honor_abort = true) {
  if (ptx::mbar_test(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_test(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
        *abort_flag = 1;
        atomicCAS(p.status, 0, kStatusTimeout);
        return false;
      }
    }
  }
}

// Whole-warp bounded wait (warp-uniform result).
__device__ __forceinline__ bool bwd_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         const BwdParams& p, bool honor_abort = true) {
  return __all_sync(0xffffffffu, bwd_wait1(bar, parity, abort_flag, p, honor_abort));
}

// Is key tile j visible to query tile qt (causal rule and block mask)?
__device__ __forceinline__ bool bwd_keep(const BwdParams& p, int bh, int qt, int j) {
  if (qt < 0 || qt >= p.nqt || j < 0 || j >= p.nkt) return false;
  if (p.causal && j * kBN > min(qt * kBM + kBM - 1, p.Nq - 1) + p.causal_off) return false;
  if (p.mask != nullptr && p.mask[((size_t)bh * p.nqt + qt) * p.nkt + j] == 0) return false;
  return true;
}

// Work unit w -> (bh, stationary tile), and the streamed tiles it visits.
template <bool kDQ>
struct BwdUnit {
  int bh, t;  // t: query tile (kDQ) or key tile
  __device__ BwdUnit(const BwdParams& p, int w) {
    const int nt = kDQ ? p.nqt : p.nkt;
    if (p.causal) {
      // kDQ: the longest query rows first; dK/dV: early key tiles are seen by
      // the most query tiles, so ascending.
      const int r = w / p.bh;
      t = kDQ ? nt - 1 - r : r;
      bh = w % p.bh;
    } else {
      bh = w / nt;
      t = w % nt;
    }
  }
  __device__ bool keep(const BwdParams& p, int u) const {
    return kDQ ? bwd_keep(p, bh, t, u) : bwd_keep(p, bh, u, t);
  }
  __device__ int end(const BwdParams& p) const { return kDQ ? p.nkt : p.nqt; }
};

// The streamed tiles a unit visits, in order: the visibility of 32 tiles is
// taken at once with one ballot, and next() is then a find-first-set (the
// issuing warp shares its sub-partition with two elementwise warps, so a
// per-tile scan of the mask and causal rule cost it ~190 cycles per tile).
// Whole warp, warp-uniform; next() returns end once the tiles are exhausted.
template <bool kDQ>
struct BwdTiles {
  int x0, e;
  uint32_t m;
  __device__ BwdTiles(const BwdParams& p, const BwdUnit<kDQ>& u) : x0(-32), e(u.end(p)), m(0u) {}
  __device__ int next(const BwdParams& p, const BwdUnit<kDQ>& u) {
    const int lane = threadIdx.x & 31;
    while (m == 0u) {
      x0 += 32;
      if (x0 >= e) return e;
      m = __ballot_sync(0xffffffffu, x0 + lane < e && u.keep(p, x0 + lane));
    }
    const int x = x0 + __ffs(m) - 1;
    m &= m - 1;
    return x;
  }
};

// C[tmem, 128 x 64] = A[smem, 128 x D] * B[smem, rows 64h.. + 64 of a tile]^T,
// both K-major.  Rows 64h.. of a 128-row tile start 64 x 128 B = 8 KB into
// each box.  Called by the whole MMA warp; one elected lane issues.
template <int D>
__device__ __forceinline__ void bwd_mma_half(uint32_t dtm, uint32_t a, uint32_t b_half) {
  constexpr uint32_t kIdesc = idesc_bf16(128, 64, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BwdCfg<D>::kBoxBytes + (kk & 3) * 32;
    if (ptx::elect_one())
      ptx::mma_ss(dtm, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b_half + off, 16, 1024),
                  kIdesc, kk > 0 ? 1u : 0u);
  }
}

// The same with A (128 x D bf16, D/2 columns) in tensor memory.
template <int D>
__device__ __forceinline__ void bwd_mma_half_ts(uint32_t dtm, uint32_t atm, uint32_t b_half) {
  constexpr uint32_t kIdesc = idesc_bf16(128, 64, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BwdCfg<D>::kBoxBytes + (kk & 3) * 32;
    if (ptx::elect_one())
      ptx::mma_ts(dtm, atm + kk * 8, smem_desc_sw128(b_half + off, 16, 1024), kIdesc, kk > 0 ? 1u : 0u);
  }
}

// C[tmem, 128 x D] (+)= A[tmem, 128 x 64 bf16 (32 columns)] * B[smem, rows
// 64h.. + 64 of a tile, used MN-major]: four K steps of 16 rows (2 KB).
template <int D>
__device__ __forceinline__ void bwd_mma_acc(uint32_t dtm, uint32_t atm, uint32_t b_half, bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    if (ptx::elect_one())
      ptx::mma_ts(dtm, atm + kk * 8, smem_desc_sw128(b_half + kk * 2048, BwdCfg<D>::kBoxBytes, 1024), kIdesc,
                  (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__device__ __forceinline__ void bwd_load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                              int row0, int bh) {
#pragma unroll
  for (int bx = 0; bx < BwdCfg<D>::kBoxes; ++bx)
    ptx::tma_load_3d(dst + bx * BwdCfg<D>::kBoxBytes, map, bar, bx * 64, row0, bh);
}

template <int D, bool kDQ>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sA = base + C::kOffA, sB = base + C::kOffB, sRing = base + C::kOffRing;
  float* vals = reinterpret_cast<float*>(base_ptr + C::kOffVals);  // [kStages][2][128]
  const BwdBars bars{base + C::kOffBar, C::kStages};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffMisc + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int items = p.bh * (kDQ ? p.nqt : p.nkt);

  // The next attention launch on the stream may start its prologue now.
  ptx::launch_dependents();
  if (threadIdx.x == 0) {
    // dQ: both elementwise warpgroups arrive once Q and dO are in tensor
    // memory; dK/dV: the producer's expect-tx arrival for the K, V tiles.
    ptx::mbar_init(bars.ab_full(), kDQ ? 256 : 1);
    ptx::mbar_init(bars.ab_empty(), 1);
    for (int s = 0; s < C::kStages; ++s) {
      // dK/dV: the producer's expect-tx arrival plus one after it stored the
      // slot's column values.
      ptx::mbar_init(bars.full(s), kDQ ? 1 : 2);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      ptx::mbar_init(bars.s_full(h), 1);
      ptx::mbar_init(bars.p_full(h), 128);
    }
    ptx::mbar_init(bars.acc_full(), 1);
    ptx::mbar_init(bars.acc_empty(), 256);
    ptx::mbar_init(bars.mma_done(), 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == kBwdLoadWarp && lane == 0) {
    ptx::prefetch_tensormap(&p.tm_q);
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_v);
    ptx::prefetch_tensormap(&p.tm_do);
  }
  if (warp == kBwdMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Everything above is this CTA's prologue; global memory is touched only
  // after the previous grid on the stream has finished (launch overlap).
  ptx::grid_dependency_wait();
  const CUtensorMap* mapA = kDQ ? &p.tm_q : &p.tm_k;
  const CUtensorMap* mapB = kDQ ? &p.tm_do : &p.tm_v;
  const CUtensorMap* mapX = kDQ ? &p.tm_k : &p.tm_q;
  const CUtensorMap* mapY = kDQ ? &p.tm_v : &p.tm_do;
  constexpr float kLog2e = 1.4426950408889634f;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------ TMA producer ---
    uint32_t it = 0, nu = 0;
    bool ok = true;
    for (int k = 0, w = unit_of_round(0); w < items && ok; w = unit_of_round(++k)) {
      const BwdUnit<kDQ> u(p, w);
      if constexpr (!kDQ) {
        ok = bwd_wait(bars.ab_empty(), (nu & 1u) ^ 1u, abort_flag, p);
        if (!ok) break;
        if (ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(bars.ab_full(), 2 * C::kTileBytes);
          bwd_load_tile<D>(sA, mapA, bars.ab_full(), u.t * kBM, u.bh);
          bwd_load_tile<D>(sB, mapB, bars.ab_full(), u.t * kBM, u.bh);
        }
        __syncwarp();
        ++nu;
      }
      BwdTiles<kDQ> tiles(p, u);
      for (int x = tiles.next(p, u); x < tiles.e && ok; x = tiles.next(p, u)) {
        const int s = it % C::kStages;
        ok = bwd_wait(bars.empty(s), ((it / C::kStages) & 1u) ^ 1u, abort_flag, p);
        if (!ok) break;
        if (ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(bars.full(s), 2 * C::kTileBytes);
          const uint32_t dst = sRing + (uint32_t)s * 2 * C::kTileBytes;
          bwd_load_tile<D>(dst, mapX, bars.full(s), x * kBM, u.bh);
          bwd_load_tile<D>(dst + C::kTileBytes, mapY, bars.full(s), x * kBM, u.bh);
        }
        if constexpr (!kDQ) {
          // Column values of query tile x: -log2(e) lse_q (-inf past Nq or
          // for a query without keys, so its P is 0) and -D_q.
          float* v = vals + s * 256;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = lane + 32 * e;
            const int q = x * kBM + c;
            float l = -INFINITY, dd = 0.f;
            if (q < p.Nq) {
              l = p.lse[(size_t)u.bh * p.Nq + q];
              dd = p.delta[(size_t)u.bh * p.Nq + q];
            }
            v[c] = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
            v[128 + c] = -dd;
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bars.full(s));
        }
        __syncwarp();
        ++it;
      }
    }
    // Drain: every load issued must land before the CTA exits.
    const uint32_t first = it > (uint32_t)C::kStages ? it - C::kStages : 0u;
    for (uint32_t r = first; r < it; ++r)
      bwd_wait(bars.full(r % C::kStages), (r / C::kStages) & 1u, abort_flag, p, false);
    if (!kDQ && nu > 0) bwd_wait(bars.ab_full(), (nu - 1) & 1u, abort_flag, p, false);
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------- MMA issuer ---
    uint32_t it = 0, nu = 0, pw0 = 0, pw1 = 0;
    bool ok = true;
    // Scores and gradient of half h of ring entry n.
    auto issue_sd = [&](int h, uint32_t n) {
      const uint32_t xb = sRing + (n % C::kStages) * 2 * C::kTileBytes;
      ptx::tc_fence_after();
      if constexpr (kDQ) {
        bwd_mma_half_ts<D>(tmem + C::s_col(h), tmem + C::kTq, xb + 8192u * h);
        bwd_mma_half_ts<D>(tmem + C::g_col(h), tmem + C::kTdo, xb + C::kTileBytes + 8192u * h);
      } else {
        bwd_mma_half<D>(tmem + C::s_col(h), sA, xb + 8192u * h);
        bwd_mma_half<D>(tmem + C::g_col(h), sB, xb + C::kTileBytes + 8192u * h);
      }
      if (ptx::elect_one()) ptx::mma_commit(bars.s_full(h));
      __syncwarp();
    };
    // Accumulation of half h of ring entry n.
    auto issue_acc = [&](int h, uint32_t n, bool accumulate) {
      const uint32_t xb = sRing + (n % C::kStages) * 2 * C::kTileBytes;
      ptx::tc_fence_after();
      if constexpr (kDQ) {
        bwd_mma_acc<D>(tmem + C::kAcc0, tmem + C::s_col(h), xb + 8192u * h, accumulate);
      } else {
        bwd_mma_acc<D>(tmem + C::kAcc0, tmem + C::s_col(h), xb + C::kTileBytes + 8192u * h, accumulate);
        bwd_mma_acc<D>(tmem + C::kAcc1, tmem + C::g_col(h), xb + 8192u * h, accumulate);
      }
      __syncwarp();
    };
    for (int k = 0, w = unit_of_round(0); w < items && ok; w = unit_of_round(++k)) {
      const BwdUnit<kDQ> u(p, w);
      ok = bwd_wait(bars.ab_full(), nu & 1u, abort_flag, p);
      if (!ok) break;
      // The previous unit's epilogue must have read the accumulators before
      // the first accumulating MMA of this unit overwrites them.
      bool need_acc_empty = nu > 0;
      BwdTiles<kDQ> tiles(p, u);
      int x = tiles.next(p, u);
      const int e = tiles.e;
      if (x < e) {
        ok = bwd_wait(bars.full(it % C::kStages), (it / C::kStages) & 1u, abort_flag, p);
        if (!ok) break;
        issue_sd(0, it);
        issue_sd(1, it);
      }
      bool first = true;
      while (x < e && ok) {
        const int xn = tiles.next(p, u);
        const bool has_next = xn < e;
        // Half 0: its P is ready -> accumulate, then half 0 of the next tile.
        ok = bwd_wait(bars.p_full(0), pw0 & 1u, abort_flag, p);
        ++pw0;
        if (!ok) break;
        if (need_acc_empty) {
          ok = bwd_wait(bars.acc_empty(), (nu - 1) & 1u, abort_flag, p);
          need_acc_empty = false;
          if (!ok) break;
        }
        issue_acc(0, it, !first);
        if (has_next) {
          ok = bwd_wait(bars.full((it + 1) % C::kStages), ((it + 1) / C::kStages) & 1u, abort_flag, p);
          if (!ok) break;
          issue_sd(0, it + 1);
        }
        // Half 1, then release the ring slot.
        ok = bwd_wait(bars.p_full(1), pw1 & 1u, abort_flag, p);
        ++pw1;
        if (!ok) break;
        issue_acc(1, it, true);
        if (ptx::elect_one()) ptx::mma_commit(bars.empty(it % C::kStages));
        __syncwarp();
        if (has_next) issue_sd(1, it + 1);
        ++it;
        first = false;
        x = xn;
      }
      if (!ok) break;
      if (need_acc_empty) {  // a unit without tiles still keeps the phases in step
        ok = bwd_wait(bars.acc_empty(), (nu - 1) & 1u, abort_flag, p);
        if (!ok) break;
      }
      if (ptx::elect_one()) {
        ptx::mma_commit(bars.acc_full());
        ptx::mma_commit(bars.ab_empty());
      }
      __syncwarp();
      ++nu;
    }
    // Drain: every MMA issued must be complete before tensor memory is freed.
    if (ptx::elect_one()) ptx::mma_commit(bars.mma_done());
    __syncwarp();
    bwd_wait(bars.mma_done(), 0, abort_flag, p, false);
  } else if (warp >= kBwdFirstEwWarp) {
    // -------------------------------------------------------- elementwise ---
    const int h = (warp - kBwdFirstEwWarp) >> 2;  // half 0 or 1
    const int r = threadIdx.x & 127;               // tensor-memory lane = tile row
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::s_col(h);
    const uint32_t tG = tmem + lane_base + C::g_col(h);
    const float c = p.scale_log2;
    uint32_t sw = 0, it = 0, nu = 0;
    bool ok = true;
    for (int k = 0, w = unit_of_round(0); w < items && ok; w = unit_of_round(++k)) {
      const BwdUnit<kDQ> u(p, w);
      const int row = u.t * kBM + r;  // query row (kDQ) or key row
      float nlse2 = -INFINITY, delta = 0.f;
      if constexpr (kDQ) {
        // This warpgroup's A operand row into tensor memory: Q (half 0) or
        // dO (half 1), zeros past Nq, once the previous unit's MMAs are done.
        ok = bwd_wait(bars.ab_empty(), (nu & 1u) ^ 1u, abort_flag, p);
        if (!ok) break;
        {
          const __nv_bfloat16* src = h == 0 ? p.q : p.dout;
          const uint4* arow = reinterpret_cast<const uint4*>(src + ((size_t)u.bh * p.Nq + (row < p.Nq ? row : 0)) * D);
          const uint32_t tA = tmem + lane_base + (h == 0 ? C::kTq : C::kTdo);
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t a[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint4 x = row < p.Nq ? arow[8 * ch + i] : make_uint4(0u, 0u, 0u, 0u);
              a[4 * i] = x.x;
              a[4 * i + 1] = x.y;
              a[4 * i + 2] = x.z;
              a[4 * i + 3] = x.w;
            }
            ptx::tmem_st32(tA + 32 * ch, a);
          }
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bars.ab_full());
        }
        // Per-row values: -log2(e) lse_i (or -inf for a row without keys),
        // D_i = dO_i . O_i, written once for the dK/dV launch.
        if (row < p.Nq) {
          const float l = p.lse[(size_t)u.bh * p.Nq + row];
          nlse2 = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
          const uint4* orow = reinterpret_cast<const uint4*>(p.o + ((size_t)u.bh * p.Nq + row) * D);
          const uint4* drow = reinterpret_cast<const uint4*>(p.dout + ((size_t)u.bh * p.Nq + row) * D);
#pragma unroll 4
          for (int i = 0; i < D / 8; ++i) {
            const uint4 a = orow[i], b = drow[i];
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              delta = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(bv[e] << 16), delta);
              delta = fmaf(__uint_as_float(av[e] & 0xFFFF0000u), __uint_as_float(bv[e] & 0xFFFF0000u), delta);
            }
          }
          if (h == 0) p.delta[(size_t)u.bh * p.Nq + row] = delta;
        }
      }
      const float ndelta = -delta;
      int ntiles = 0;
      BwdTiles<kDQ> tiles(p, u);
      for (int x = tiles.next(p, u); x < tiles.e && ok; x = tiles.next(p, u)) {
        ok = bwd_wait(bars.s_full(h), sw & 1u, abort_flag, p);
        ++sw;
        if (!ok) break;
        ptx::tc_fence_after();
        const int col0 = x * kBM + 64 * h;  // first key (kDQ) or query of this half
        if constexpr (kDQ) {
          // Visible keys of this row within the half: c <= lim.
          int last = p.Nk - 1;
          if (p.causal) last = min(last, row + p.causal_off);
          const int lim = last - col0;
          // All 64 scores and 64 gradients in one round trip.
          uint32_t rs[2][32], rp[2][32];
          ptx::tmem_ld32(tS, rs[0]);
          ptx::tmem_ld32(tS + 32, rs[1]);
          ptx::tmem_ld32(tG, rp[0]);
          ptx::tmem_ld32(tG + 32, rp[1]);
          ptx::tmem_wait_ld();
          uint32_t pk[32];
          // Pairs of columns with packed f32x2 arithmetic; the mask only on
          // tiles that reach the diagonal or the end of the keys.
          auto body = [&](auto masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = 2 * e;
              float x0, x1, p0, p1, g0, g1, d0, d1;
              ptx::fma2(x0, x1, __uint_as_float(rs[col >> 5][col & 31]),
                        __uint_as_float(rs[col >> 5][(col & 31) + 1]), c, c, nlse2, nlse2);
              p0 = ptx::ex2(x0);
              p1 = ptx::ex2(x1);
              if constexpr (decltype(masked)::value) {
                p0 = col <= lim ? p0 : 0.f;
                p1 = col + 1 <= lim ? p1 : 0.f;
              }
              ptx::add2(g0, g1, __uint_as_float(rp[col >> 5][col & 31]),
                        __uint_as_float(rp[col >> 5][(col & 31) + 1]), ndelta, ndelta);
              ptx::mul2(d0, d1, p0, p1, g0, g1);
              pk[e] = ptx::pack_bf16x2(d0, d1);
            }
          };
          if (__all_sync(0xffffffffu, lim >= 63)) body(std::false_type{});
          else body(std::true_type{});
          ptx::tmem_st32(tS, pk);  // dS over S columns [0, 32)
        } else {
          // Visible queries of this key row within the half: c >= lo.
          const int lo = p.causal ? row - p.causal_off - col0 : INT_MIN;
          const float* v = vals + (it % C::kStages) * 256 + 64 * h;
          // 32 columns at a time: P^T over S^T columns [16 ch, 16 ch + 16),
          // dS^T likewise over dP^T (both already read).  Four columns per
          // step: their -log2(e) lse and -D as float4 (broadcast shared-memory
          // reads), packed f32x2 arithmetic; the mask only on tiles that reach
          // the causal diagonal.
          const bool masked = !__all_sync(0xffffffffu, lo <= 0);
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t rs[32], rp[32];
            ptx::tmem_ld32(tS + 32 * ch, rs);
            ptx::tmem_ld32(tG + 32 * ch, rp);
            ptx::tmem_wait_ld();
            uint32_t pp[16], pd[16];
            auto body = [&](auto mtag) {
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const int k = 4 * e4;
                const int col = 32 * ch + k;
                const float4 nl = *reinterpret_cast<const float4*>(v + col);
                const float4 nd = *reinterpret_cast<const float4*>(v + 128 + col);
                const float nla[4] = {nl.x, nl.y, nl.z, nl.w}, nda[4] = {nd.x, nd.y, nd.z, nd.w};
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  float x0, x1, p0, p1, g0, g1, d0, d1;
                  ptx::fma2(x0, x1, __uint_as_float(rs[k + 2 * j]), __uint_as_float(rs[k + 2 * j + 1]), c, c,
                            nla[2 * j], nla[2 * j + 1]);
                  p0 = ptx::ex2(x0);
                  p1 = ptx::ex2(x1);
                  if constexpr (decltype(mtag)::value) {
                    p0 = col + 2 * j >= lo ? p0 : 0.f;
                    p1 = col + 2 * j + 1 >= lo ? p1 : 0.f;
                  }
                  ptx::add2(g0, g1, __uint_as_float(rp[k + 2 * j]), __uint_as_float(rp[k + 2 * j + 1]),
                            nda[2 * j], nda[2 * j + 1]);
                  ptx::mul2(d0, d1, p0, p1, g0, g1);
                  pp[2 * e4 + j] = ptx::pack_bf16x2(p0, p1);
                  pd[2 * e4 + j] = ptx::pack_bf16x2(d0, d1);
                }
              }
            };
            if (masked) body(std::true_type{});
            else body(std::false_type{});
            ptx::tmem_st16(tS + 16 * ch, pp);
            ptx::tmem_st16(tG + 16 * ch, pd);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bars.p_full(h));
        ++it;
        ++ntiles;
      }
      if (!ok) break;
      // ------------------------------------------------------- epilogue ---
      ok = bwd_wait(bars.acc_full(), nu & 1u, abort_flag, p);
      ++nu;
      if (!ok) break;
      ptx::tc_fence_after();
      const int nrows = kDQ ? p.Nq : p.Nk;
      const bool in_range = row < nrows;
      // kDQ: half h stores columns [h D/2, (h+1) D/2) of dQ.  Else half 0
      // stores dV, half 1 dK.
      constexpr int kCols = kDQ ? D / 2 : D;
      __nv_bfloat16* dst = kDQ ? p.dq : (h == 0 ? p.dv : p.dk);
      const uint32_t tAcc = tmem + lane_base + (kDQ ? C::kAcc0 + h * (D / 2) : (h == 0 ? C::kAcc0 : C::kAcc1));
      const float f = (kDQ || h == 1) ? p.scale : 1.f;
      uint4* out = reinterpret_cast<uint4*>(dst + ((size_t)u.bh * nrows + (in_range ? row : 0)) * D +
                                            (kDQ ? h * (D / 2) : 0));
#pragma unroll 1
      for (int ch = 0; ch < kCols / 32; ++ch) {
        uint32_t t[32];
        if (ntiles > 0) {
          ptx::tmem_ld32(tAcc + 32 * ch, t);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) t[e] = 0u;
        }
        uint32_t pkd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pkd[e] = ptx::pack_bf16x2(__uint_as_float(t[2 * e]) * f, __uint_as_float(t[2 * e + 1]) * f);
        if (in_range) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            out[ch * 4 + v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bars.acc_empty());
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
