// Backward pass of the fused attention for B200 (sm_100a): dQ, dK, dV.
//
// The score matrix is not stored by the forward pass; it is recomputed here
// from Q, K and the forward's logsumexp ("理解 Flash Attention", section
// "瓦片注意力计算": S is needed for backpropagation and recomputed there, which
// keeps memory O(n)).  With P_ij = exp(scale q_i.k_j - lse_i) over visible keys:
//   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Two kernels, no atomics:
//  * fa_bwd_dq_kernel, stationary on a 128-row query tile: per visible key
//    tile j, S = Q K_j^T and dP = dO V_j^T (tcgen05, fp32 in tensor memory),
//    the elementwise dS (one thread per query row, bf16 written over S), then
//    dQ += dS K_j (A operand read from tensor memory).  It also writes D_i to
//    the workspace for the second kernel.
//  * fa_bwd_dkdv_kernel, stationary on a 128-key tile: per query tile i that
//    sees it, S^T = K Q_i^T and dP^T = V dO_i^T (one thread per key row), P^T
//    and dS^T in bf16 over them, then dV += P^T dO_i and dK += dS^T Q_i.
//
// Each CTA is one warpgroup.  All four warps do the elementwise work; the
// elected lane of warp 0 also issues the TMA loads and the MMAs.  Per tile the
// order is: S/dP MMAs -> elementwise -> accumulating MMA(s), with the next
// tile's S/dP MMAs queued right behind the accumulating ones.  The ring holds
// two tiles ahead.  Every barrier wait is bounded as in the forward kernel.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

struct BwdParams {
  CUtensorMap tm_q;   // [B*H][Nq][D] bf16, box 64 x 128 x 1, 128B swizzle
  CUtensorMap tm_k;   // [B*H][Nk][D]
  CUtensorMap tm_v;   // [B*H][Nk][D]
  CUtensorMap tm_do;  // [B*H][Nq][D]
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;  // [B*H][Nq]
  float* delta;      // [B*H][Nq], written by the dQ kernel
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const uint8_t* mask;  // nullptr or [B*H][nqt][nkt]
  int Nq, Nk, nqt, nkt, causal_off, bh, causal;
  float scale, scale_log2;
  unsigned long long timeout_ns;
  int* status;
};

constexpr int kBwdThreads = 128;

template <int D>
struct BwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kPairs = 2;  // ring depth, in (two-tile) steps
  // Stationary tiles A, B (dQ: Q, dO; dK/dV: K, V), then the ring of
  // kPairs x {first, second} streamed tiles (dQ: K_j, V_j; dK/dV: Q_i, dO_i).
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kTileBytes;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + 2 * kPairs * kTileBytes;
  // ab_full, full[kPairs], empty[kPairs], sd_full, acc_full
  static constexpr int kNumBars = 1 + 2 * kPairs + 2;
  static constexpr int kOffVals = (kOffBar + kNumBars * 8 + 15) / 16 * 16;  // 2 x 128 floats
  static constexpr int kOffMisc = kOffVals + 2 * 128 * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};

struct BwdBars {
  uint32_t ab_full, sd_full, acc_full, full0, empty0;
  __device__ uint32_t full(int s) const { return full0 + 8u * s; }
  __device__ uint32_t empty(int s) const { return empty0 + 8u * s; }
};

// Bounded wait by a whole warp (warp-uniform result).
__device__ __forceinline__ bool bwd_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         const BwdParams& p, bool honor_abort = true) {
  bool ok = ptx::mbar_test(bar, parity);
  if (!ok) {
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ptx::mbar_test(bar, parity)) {
        ok = true;
        break;
      }
      if ((it & 31u) == 0) {
        if (honor_abort && *abort_flag) break;
        if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
          *abort_flag = 1;
          atomicCAS(p.status, 0, kStatusTimeout);
          break;
        }
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Is key tile j visible to query tile qt (causal rule and block mask)?
__device__ __forceinline__ bool bwd_keep(const BwdParams& p, int bh, int qt, int j) {
  if (qt < 0 || qt >= p.nqt || j < 0 || j >= p.nkt) return false;
  if (p.causal && j * kBN > min(qt * kBM + kBM - 1, p.Nq - 1) + p.causal_off) return false;
  if (p.mask != nullptr && p.mask[((size_t)bh * p.nqt + qt) * p.nkt + j] == 0) return false;
  return true;
}

// CTA-wide barrier of the 128 threads (named barrier 1; 0 is __syncthreads).
__device__ __forceinline__ void bwd_sync() { ptx::named_barrier(1, kBwdThreads); }

template <int D>
__device__ __forceinline__ void bwd_setup(uint8_t* smem_raw, uint32_t& base, uint8_t*& base_ptr,
                                          BwdBars& bars, uint32_t*& tmem_slot,
                                          volatile int*& abort_flag) {
  using C = BwdCfg<D>;
  const uint32_t raw = ptx::smem_u32(smem_raw);
  base = (raw + 1023u) & ~1023u;
  base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + C::kOffBar;
  bars.ab_full = bar0;
  bars.full0 = bar0 + 8;
  bars.empty0 = bar0 + 8 + 8 * C::kPairs;
  bars.sd_full = bar0 + 8 + 16 * C::kPairs;
  bars.acc_full = bars.sd_full + 8;
  tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffMisc);
  abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffMisc + 4);
  if (threadIdx.x == 0) {
    ptx::mbar_init(bars.ab_full, 1);
    for (int s = 0; s < C::kPairs; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);
    }
    ptx::mbar_init(bars.sd_full, 1);
    ptx::mbar_init(bars.acc_full, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
  }
  if (threadIdx.x < 32) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
}

// Load a 128-row tile (rows row0.. of head bh) of `map` into `dst` on `bar`.
template <int D>
__device__ __forceinline__ void bwd_load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                              int row0, int bh) {
#pragma unroll
  for (int bx = 0; bx < BwdCfg<D>::kBoxes; ++bx)
    ptx::tma_load_3d(dst + bx * BwdCfg<D>::kBoxBytes, map, bar, bx * 64, row0, bh);
}

// C[tmem] (+)= A[smem, K-major] * B[smem, K-major]^T over K = D (two 128-row tiles).
template <int D>
__device__ __forceinline__ void bwd_mma_ss(uint32_t dtm, uint32_t a, uint32_t b) {
  constexpr uint32_t kIdesc = idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BwdCfg<D>::kBoxBytes + (kk & 3) * 32;
    ptx::mma_ss(dtm, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), kIdesc,
                kk > 0 ? 1u : 0u);
  }
}

// C[tmem, 128 x D] (+)= A[tmem, 128 x 128 bf16] * B[smem tile, 128 rows x D, used MN-major].
template <int D>
__device__ __forceinline__ void bwd_mma_ts(uint32_t dtm, uint32_t atm, uint32_t b, bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    ptx::mma_ts(dtm, atm + kk * 8, smem_desc_sw128(b + kk * 2048, BwdCfg<D>::kBoxBytes, 1024), kIdesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

// Drain the MMA pipe and free tensor memory (end of kernel, all threads).
__device__ __forceinline__ void bwd_teardown(uint32_t tmem, const BwdBars& bars,
                                             volatile int* abort_flag, const BwdParams& p,
                                             uint32_t acc_count) {
  if (threadIdx.x < 32) {
    if (ptx::elect_one()) ptx::mma_commit(bars.acc_full);
    __syncwarp();
    bwd_wait(bars.acc_full, acc_count & 1u, abort_flag, p, false);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Ring bookkeeping of the leader warp: streamed tile pair n goes to slot
// n % kPairs; its load is issued once the previous occupant was released.
template <int D>
struct BwdRing {
  uint32_t loads = 0;  // pairs loaded
  uint32_t uses = 0;   // pairs consumed
  __device__ int slot(uint32_t n) const { return n % BwdCfg<D>::kPairs; }
  __device__ uint32_t phase(uint32_t n) const { return (n / BwdCfg<D>::kPairs) & 1u; }
};

// Leader warp: load streamed pair (first, second) of tile `row0` into the
// ring (waiting for the slot to be released), returns false on abort.
template <int D>
__device__ __forceinline__ bool bwd_ring_load(BwdRing<D>& r, const BwdBars& bars, uint32_t sRing,
                                              const CUtensorMap* m1, const CUtensorMap* m2,
                                              int row0, int bh, volatile int* abort_flag,
                                              const BwdParams& p) {
  using C = BwdCfg<D>;
  const int s = r.slot(r.loads);
  if (!bwd_wait(bars.empty(s), r.phase(r.loads) ^ 1u, abort_flag, p)) return false;
  if (ptx::elect_one()) {
    ptx::mbar_arrive_expect_tx(bars.full(s), 2 * C::kTileBytes);
    const uint32_t dst = sRing + (uint32_t)s * 2 * C::kTileBytes;
    bwd_load_tile<D>(dst, m1, bars.full(s), row0, bh);
    bwd_load_tile<D>(dst + C::kTileBytes, m2, bars.full(s), row0, bh);
  }
  __syncwarp();
  ++r.loads;
  return true;
}

// ---------------------------------------------------------------- dQ ---
//
// Tensor memory: S [0,128) (dS in bf16 over its first 64 columns),
// dP [128,256), dQ accumulator [256,256+D).
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base;
  uint8_t* base_ptr;
  BwdBars bars;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  bwd_setup<D>(smem_raw, base, base_ptr, bars, tmem_slot, abort_flag);
  const uint32_t tmem = *tmem_slot;
  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t sQ = base + C::kOffA, sDO = base + C::kOffB, sRing = base + C::kOffRing;
  constexpr uint32_t kS = 0, kDP = 128, kDQ = 256;
  const float c = p.scale_log2;
  constexpr float kLog2e = 1.4426950408889634f;

  BwdRing<D> ring;
  uint32_t ab = 0, sd = 0, acc = 0;
  bool ok = true;
  const int items = p.bh * p.nqt;
  for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
    int bh, qt;
    if (p.causal) {  // longest rows first
      qt = p.nqt - 1 - w / p.bh;
      bh = w % p.bh;
    } else {
      bh = w / p.nqt;
      qt = w % p.nqt;
    }
    const int row = qt * kBM + tid;
    const bool in_range = row < p.Nq;
    // Visible key tiles: j walks them in order; `next` finds the following one.
    auto next = [&](int j) {
      for (++j; j < p.nkt; ++j)
        if (bwd_keep(p, bh, qt, j)) return j;
      return p.nkt;
    };
    const int j_first = next(-1);
    // Stationary Q and dO, and the first two streamed tiles.
    if (warp == 0) {
      if (ptx::elect_one()) {
        ptx::mbar_arrive_expect_tx(bars.ab_full, 2 * C::kTileBytes);
        bwd_load_tile<D>(sQ, &p.tm_q, bars.ab_full, qt * kBM, bh);
        bwd_load_tile<D>(sDO, &p.tm_do, bars.ab_full, qt * kBM, bh);
      }
      __syncwarp();
      int jl = j_first;
      for (int n = 0; n < C::kPairs && jl < p.nkt && ok; ++n, jl = next(jl))
        ok = bwd_ring_load<D>(ring, bars, sRing, &p.tm_k, &p.tm_v, jl * kBN, bh, abort_flag, p);
    }
    // Per-row values: -log2(e) lse_i (or -inf for a row without keys), D_i.
    float nlse2 = -INFINITY, delta = 0.f;
    if (in_range) {
      const float l = p.lse[(size_t)bh * p.Nq + row];
      nlse2 = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
      const uint4* orow = reinterpret_cast<const uint4*>(p.o + ((size_t)bh * p.Nq + row) * D);
      const uint4* drow = reinterpret_cast<const uint4*>(p.dout + ((size_t)bh * p.Nq + row) * D);
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
      p.delta[(size_t)bh * p.Nq + row] = delta;
    }
    ok = __all_sync(0xffffffffu, ok);
    bwd_sync();
    if (!__syncthreads_and(ok)) break;
    ok = bwd_wait(bars.ab_full, ab & 1u, abort_flag, p);
    ++ab;
    ok = __syncthreads_and(ok);  // every loop exit below is CTA-uniform
    int ntiles = 0;
    for (int j = j_first; j < p.nkt && ok; j = next(j)) {
      const int s = ring.slot(ring.uses);
      const uint32_t kbase = sRing + (uint32_t)s * 2 * C::kTileBytes;
      if (j == j_first && warp == 0) {  // S and dP of the first tile
        ok = bwd_wait(bars.full(s), ring.phase(ring.uses), abort_flag, p);
        ptx::tc_fence_after();
        if (ok && ptx::elect_one()) {
          bwd_mma_ss<D>(tmem + kS, sQ, kbase);
          bwd_mma_ss<D>(tmem + kDP, sDO, kbase + C::kTileBytes);
          ptx::mma_commit(bars.sd_full);
        }
        __syncwarp();
      }
      ok = bwd_wait(bars.sd_full, sd & 1u, abort_flag, p) && ok;
      ++sd;
      if (!__syncthreads_and(ok)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // dS = P o (dP - D) for this row, 32 key columns at a time; the bf16 dS
      // of chunk ch lands in S columns [16 ch, 16 ch + 16), which earlier
      // chunks have already read.
      int lim = 127;  // last visible key column of this tile
      if (p.causal) lim = min(lim, row + p.causal_off - j * kBN);
      lim = min(lim, p.Nk - j * kBN - 1);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rs[32], rp[32];
        ptx::tmem_ld32(tmem + lane_base + kS + 32 * ch, rs);
        ptx::tmem_ld32(tmem + lane_base + kDP + 32 * ch, rp);
        ptx::tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float ds[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int col = 32 * ch + 2 * e + h;
            const float pr = col <= lim ? ptx::ex2(fmaf(__uint_as_float(rs[2 * e + h]), c, nlse2)) : 0.f;
            ds[h] = pr * (__uint_as_float(rp[2 * e + h]) - delta);
          }
          pk[e] = ptx::pack_bf16x2(ds[0], ds[1]);
        }
        ptx::tmem_st16(tmem + lane_base + kS + 16 * ch, pk);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      bwd_sync();
      // dQ += dS K_j; then the next tile's S and dP; then refill the ring.
      if (warp == 0) {
        ptx::tc_fence_after();
        const uint32_t un = ring.uses;
        if (ptx::elect_one()) {
          bwd_mma_ts<D>(tmem + kDQ, tmem + kS, kbase, ntiles > 0);
          ptx::mma_commit(bars.empty(s));
        }
        __syncwarp();
        ++ring.uses;
        const int jn = next(j);
        if (jn < p.nkt) {
          const int s2 = ring.slot(ring.uses);
          ok = bwd_wait(bars.full(s2), ring.phase(ring.uses), abort_flag, p);
          ptx::tc_fence_after();
          const uint32_t kb2 = sRing + (uint32_t)s2 * 2 * C::kTileBytes;
          if (ok && ptx::elect_one()) {
            bwd_mma_ss<D>(tmem + kS, sQ, kb2);
            bwd_mma_ss<D>(tmem + kDP, sDO, kb2 + C::kTileBytes);
            ptx::mma_commit(bars.sd_full);
          }
          __syncwarp();
          // Refill: the tile after next, into the slot released by dQ above.
          const int jf = next(jn);
          if (ok && jf < p.nkt && ring.loads < un + 1 + C::kPairs)
            ok = bwd_ring_load<D>(ring, bars, sRing, &p.tm_k, &p.tm_v, jf * kBN, bh, abort_flag, p);
        }
      } else {
        ring.uses += 1;
      }
      ++ntiles;
      ok = __syncthreads_and(ok);  // warp 0's refill result, for everyone
    }
    if (!__syncthreads_and(ok)) break;
    // Epilogue: dQ = scale * accumulator (zero when no key tile is visible).
    if (warp == 0) {
      if (ptx::elect_one()) ptx::mma_commit(bars.acc_full);
      __syncwarp();
    }
    ok = bwd_wait(bars.acc_full, acc & 1u, abort_flag, p);
    ++acc;
    if (!__syncthreads_and(ok)) break;
    ptx::tc_fence_after();
    uint4* out = reinterpret_cast<uint4*>(p.dq + ((size_t)bh * p.Nq + (in_range ? row : 0)) * D);
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t t[32];
      if (ntiles > 0) {
        ptx::tmem_ld32(tmem + lane_base + kDQ + 32 * ch, t);
        ptx::tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) t[e] = 0u;
      }
      uint32_t pkd[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pkd[e] = ptx::pack_bf16x2(__uint_as_float(t[2 * e]) * p.scale, __uint_as_float(t[2 * e + 1]) * p.scale);
      if (in_range) {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          out[ch * 4 + v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
      }
    }
    ptx::tc_fence_before();
    bwd_sync();  // the accumulator is read before the next unit overwrites it
  }
  bwd_teardown(tmem, bars, abort_flag, p, acc);
}

// ------------------------------------------------------------- dK, dV ---
//
// Tensor memory: S^T [0,128) (P^T in bf16 over its first 64 columns),
// dP^T [128,256) (dS^T in bf16 over its first 64 columns), dV [256,256+D),
// dK [384,384+D).  One thread per key row; columns are queries.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base;
  uint8_t* base_ptr;
  BwdBars bars;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  bwd_setup<D>(smem_raw, base, base_ptr, bars, tmem_slot, abort_flag);
  const uint32_t tmem = *tmem_slot;
  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t sK = base + C::kOffA, sV = base + C::kOffB, sRing = base + C::kOffRing;
  float* nlse2s = reinterpret_cast<float*>(base_ptr + C::kOffVals);  // -log2(e) lse_q of the tile
  float* deltas = nlse2s + 128;                                       // D_q of the tile
  constexpr uint32_t kST = 0, kDPT = 128, kDV = 256, kDK = 384;
  const float c = p.scale_log2;
  constexpr float kLog2e = 1.4426950408889634f;

  BwdRing<D> ring;
  uint32_t ab = 0, sd = 0, acc = 0;
  bool ok = true;
  const int items = p.bh * p.nkt;
  for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
    int bh, kt;
    if (p.causal) {  // early key tiles are seen by the most query tiles: first
      kt = w / p.bh;
      bh = w % p.bh;
    } else {
      bh = w / p.nkt;
      kt = w % p.nkt;
    }
    const int r = kt * kBN + tid;  // this thread's key row
    const bool in_range = r < p.Nk;
    auto next = [&](int i) {
      for (++i; i < p.nqt; ++i)
        if (bwd_keep(p, bh, i, kt)) return i;
      return p.nqt;
    };
    const int i_first = next(-1);
    if (warp == 0) {
      if (ptx::elect_one()) {
        ptx::mbar_arrive_expect_tx(bars.ab_full, 2 * C::kTileBytes);
        bwd_load_tile<D>(sK, &p.tm_k, bars.ab_full, kt * kBN, bh);
        bwd_load_tile<D>(sV, &p.tm_v, bars.ab_full, kt * kBN, bh);
      }
      __syncwarp();
      int il = i_first;
      for (int n = 0; n < C::kPairs && il < p.nqt && ok; ++n, il = next(il))
        ok = bwd_ring_load<D>(ring, bars, sRing, &p.tm_q, &p.tm_do, il * kBM, bh, abort_flag, p);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!__syncthreads_and(ok)) break;
    ok = bwd_wait(bars.ab_full, ab & 1u, abort_flag, p);
    ++ab;
    ok = __syncthreads_and(ok);  // every loop exit below is CTA-uniform
    int ntiles = 0;
    for (int i = i_first; i < p.nqt && ok; i = next(i)) {
      const int s = ring.slot(ring.uses);
      const uint32_t qbase = sRing + (uint32_t)s * 2 * C::kTileBytes;
      // Column values of this query tile.
      {
        const int q = i * kBM + tid;
        float l = -INFINITY, dd = 0.f;
        if (q < p.Nq) {
          l = p.lse[(size_t)bh * p.Nq + q];
          dd = p.delta[(size_t)bh * p.Nq + q];
        }
        nlse2s[tid] = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
        deltas[tid] = dd;
      }
      if (i == i_first && warp == 0) {  // S^T and dP^T of the first tile
        ok = bwd_wait(bars.full(s), ring.phase(ring.uses), abort_flag, p);
        ptx::tc_fence_after();
        if (ok && ptx::elect_one()) {
          bwd_mma_ss<D>(tmem + kST, sK, qbase);
          bwd_mma_ss<D>(tmem + kDPT, sV, qbase + C::kTileBytes);
          ptx::mma_commit(bars.sd_full);
        }
        __syncwarp();
      }
      ok = bwd_wait(bars.sd_full, sd & 1u, abort_flag, p) && ok;
      ++sd;
      if (!__syncthreads_and(ok)) {  // also publishes the column values
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // P^T and dS^T of this key row, 32 query columns at a time.
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rs[32], rp[32];
        ptx::tmem_ld32(tmem + lane_base + kST + 32 * ch, rs);
        ptx::tmem_ld32(tmem + lane_base + kDPT + 32 * ch, rp);
        ptx::tmem_wait_ld();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float pv[2], dv[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int col = 32 * ch + 2 * e + h;
            const int q = i * kBM + col;
            const bool vis = in_range && q < p.Nq && (!p.causal || r <= q + p.causal_off);
            const float pr = vis ? ptx::ex2(fmaf(__uint_as_float(rs[2 * e + h]), c, nlse2s[col])) : 0.f;
            pv[h] = pr;
            dv[h] = pr * (__uint_as_float(rp[2 * e + h]) - deltas[col]);
          }
          pp[e] = ptx::pack_bf16x2(pv[0], pv[1]);
          pd[e] = ptx::pack_bf16x2(dv[0], dv[1]);
        }
        ptx::tmem_st16(tmem + lane_base + kST + 16 * ch, pp);
        ptx::tmem_st16(tmem + lane_base + kDPT + 16 * ch, pd);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      bwd_sync();
      // dV += P^T dO_i, dK += dS^T Q_i; then the next tile's S^T, dP^T; refill.
      if (warp == 0) {
        ptx::tc_fence_after();
        const uint32_t un = ring.uses;
        if (ptx::elect_one()) {
          bwd_mma_ts<D>(tmem + kDV, tmem + kST, qbase + C::kTileBytes, ntiles > 0);
          bwd_mma_ts<D>(tmem + kDK, tmem + kDPT, qbase, ntiles > 0);
          ptx::mma_commit(bars.empty(s));
        }
        __syncwarp();
        ++ring.uses;
        const int in = next(i);
        if (in < p.nqt) {
          const int s2 = ring.slot(ring.uses);
          ok = bwd_wait(bars.full(s2), ring.phase(ring.uses), abort_flag, p);
          ptx::tc_fence_after();
          const uint32_t qb2 = sRing + (uint32_t)s2 * 2 * C::kTileBytes;
          if (ok && ptx::elect_one()) {
            bwd_mma_ss<D>(tmem + kST, sK, qb2);
            bwd_mma_ss<D>(tmem + kDPT, sV, qb2 + C::kTileBytes);
            ptx::mma_commit(bars.sd_full);
          }
          __syncwarp();
          const int iff = next(in);
          if (ok && iff < p.nqt && ring.loads < un + 1 + C::kPairs)
            ok = bwd_ring_load<D>(ring, bars, sRing, &p.tm_q, &p.tm_do, iff * kBM, bh, abort_flag, p);
        }
      } else {
        ring.uses += 1;
      }
      ++ntiles;
      // Column values are rewritten by the next tile; warp 0's refill result.
      ok = __syncthreads_and(ok);
    }
    if (!__syncthreads_and(ok)) break;
    if (warp == 0) {
      if (ptx::elect_one()) ptx::mma_commit(bars.acc_full);
      __syncwarp();
    }
    ok = bwd_wait(bars.acc_full, acc & 1u, abort_flag, p);
    ++acc;
    if (!__syncthreads_and(ok)) break;
    ptx::tc_fence_after();
    // Epilogue: dV and scale * dK for this key row (zero when no query sees it).
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      __nv_bfloat16* dst = which == 0 ? p.dv : p.dk;
      const float f = which == 0 ? 1.f : p.scale;
      const uint32_t col0 = which == 0 ? kDV : kDK;
      uint4* out = reinterpret_cast<uint4*>(dst + ((size_t)bh * p.Nk + (in_range ? r : 0)) * D);
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t t[32];
        if (ntiles > 0) {
          ptx::tmem_ld32(tmem + lane_base + col0 + 32 * ch, t);
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
    }
    ptx::tc_fence_before();
    bwd_sync();
  }
  bwd_teardown(tmem, bars, abort_flag, p, acc);
}

}  // namespace fa
