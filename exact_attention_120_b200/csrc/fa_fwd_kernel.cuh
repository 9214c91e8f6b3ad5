// Fused exact-attention forward kernel for B200 (sm_100a).
//
// What it computes (per batch b, head h, query row i):
//   O_i = sum_j softmax_j(scale * q_i . k_j) v_j over the visible keys j, and
//   lse_i = ln sum_j exp(scale * q_i . k_j)
// in one pass over the keys with the online softmax (AllenY's blog,
// "FlashAttention" post, sections "从3-pass到2-pass" and "FlashAttention";
// wmrh.cn FlashAttention article, "2.2 把 Online Softmax 嵌入注意力": one Q
// block stays put while every K/V block streams past, with per-row running
// max m, denominator l and an output accumulator corrected when m grows).
// The N x N scores live only in tensor memory.
//
// Work unit: a pair of 128-row query tiles (2p, 2p+1) of one (b, h) -- the
// Q-block-stationary split of "理解 Flash Attention" ("算法概述": one job per Q
// block, streaming all of K and V), with two Q blocks sharing each K/V tile.
// The grid is persistent: CTA c takes one unit of every round of gridDim.x
// units, in the order unit_of_round gives.
//
// Instantiations: Cfg<D, fp8> for head dim 64 or 128 with bf16 inputs, or
// d = 128 with e4m3 inputs (tcgen05 kind::f8f6f4); kVarlen for packed
// variable-length batches.  One source, the same roles and barriers.
//
// Warp roles (384 threads, one CTA per SM, 512 tensor-memory columns):
//   warp  0    MMA issue (warp-uniform loop, one elected lane issues):
//              S_q = Q_q K_j^T and O_q += P_q V_j
//   warp  1    TMA producer: Q tiles, then K_j, V_j through a ring in smem
//   warps 2-3  idle
//   warps 4-7  softmax for query tile 2p   (thread t owns row t of the tile)
//   warps 8-11 softmax for query tile 2p+1
// The issuing warps have the lowest ids: warp schedulers favour them over the
// long-running softmax warps that share their SM sub-partitions.
//
// Tensor memory (fp32 columns, lane = tile row):
//   S_0 [0,128)  S_1 [128,256)  O_0 [256,256+D)  O_1 [384,384+D)
//   d = 128: P_q (bf16 pairs in 64 columns, or e4m3 quads in 32) overwrites
//   the start of S_q once the softmax has read S_q into registers; the PV
//   MMA reads P_q from there.  d = 64: O_q takes 64 columns and P_q gets its
//   own ([384,448), [448,512)), so the next S_q can run during the softmax.
//
// Online softmax in base 2: with c = scale * log2(e), each row keeps a
// reference max m_ref (in units of c * score) and l = sum 2^(c s - m_ref).
// The reference is moved (and O, l rescaled by 2^(m_old - m_new), the
// concatenation rule of "理解 Flash Attention", "瓦片注意力计算") only when the
// tile max exceeds it by more than Cfg::kRescale (2^8 for bf16 P, so p <= 2^8;
// e4m3 P moves at 2^4 with a 2^4 shift, see Cfg).  l sums the rounded p that
// the PV MMA consumes, so O / l is an exact convex combination of V rows.
//
// Every wait on an mbarrier is bounded (globaltimer); on expiry the CTA
// records FA_ERR_DEVICE_TIMEOUT, all roles leave their loops, in-flight TMA
// loads and MMAs are drained and tensor memory is released before exit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace fa {

constexpr int kBM = 128;  // query rows per tile (= MMA M)
constexpr int kBN = 128;  // keys per tile (= mask block)
constexpr int kThreads = 384;
constexpr int kMmaWarp = 0;
constexpr int kLoadWarp = 1;
constexpr int kFirstSoftmaxWarp = 4;
constexpr uint32_t kTmemCols = 512;
constexpr int kStatusTimeout = 4;  // == FA_ERR_DEVICE_TIMEOUT
// Variable-length batches: sequences per launch, bounded by the shared-memory
// table of their first work units (larger batches take several launches).
constexpr int kMaxVarlenSeqs = 4096;

struct KernelParams {
  CUtensorMap tm_q;  // 3-D maps over [B*H][N][D] bf16, box 64 x 128 x 1, 128B swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* o;
  int o_v8;  // o is 32-byte aligned: the epilogue may use 32-byte stores
  float* lse;
  const uint8_t* mask;  // nullptr or [B*H][nqt][nkt]
  int Nq;          // query rows per head
  int Nk;          // keys per head
  int nqt;         // query tiles per head
  int nkt;         // key tiles per head
  int causal_off;  // Nk - Nq: key j is visible to query i iff j <= i + causal_off
  int npairs;      // work units per head
  int bh;      // B * H
  int group;   // causal order: heads per group (their K/V together fit in L2)
  int items;   // bh * npairs
  int causal;
  float scale_log2;  // scale * log2(e) (8-bit inputs: times the Q and K dequantisation scales)
  float o_scale;     // multiplies O: 1, or the V dequantisation scale for 8-bit inputs
  unsigned long long timeout_ns;
  int* status;  // device status word
  // Test hook of the failure-detection test: when set, the TMA producer issues
  // nothing, so the first barrier wait of the MMA issuer can never complete and
  // must end through its time limit.  Always 0 on the production entry points.
  int starve_producer;
  // Split key ranges (flash-decoding style): a work unit covers key tiles
  // [split * kt_per_split, (split + 1) * kt_per_split).  With splits > 1 the
  // epilogue writes the unit's normalised fp32 partial O and its partial lse to
  // the caller's workspace instead of O and lse; fa_combine_kernel merges them.
  int splits;
  int kt_per_split;
  float* part_o;    // [splits][B*H*Nq][D]
  float* part_lse;  // [splits][B*H*Nq]
  // Variable-length batches (the kernel's kVarlen instantiation): q, k, v and o
  // are packed tokens [T][H][D]; sequence b owns token rows
  // [cu_q[b], cu_q[b+1]) of the queries and [cu_k[b], cu_k[b+1]) of the keys;
  // lse is [H][total_q].  Nq / Nk / nqt / nkt then hold the maxima over the
  // batch and only bound the work grid.
  const int* cu_q;
  const int* cu_k;
  int heads;
  int total_q;
  int total_k;
  int nseq;        // sequences of this launch (at most kMaxVarlenSeqs)
  int group_keys;  // causal order: keys whose K/V of one head fit the L2 share of a head group
};

// Sizes of the (b, h) problem a work unit belongs to.  Dense batches: every
// head has the kernel-wide sizes, read straight from the kernel parameters.
// Variable-length batches: read from the sequence offsets, clamped to
// [0, total] and made non-decreasing, so that any offsets keep every access
// inside the buffers.
struct SeqDense {
  const KernelParams& p;
  __device__ int nq() const { return p.Nq; }
  __device__ int nk() const { return p.Nk; }
  __device__ int nqt() const { return p.nqt; }
  __device__ int nkt() const { return p.nkt; }
  __device__ int causal_off() const { return p.causal_off; }  // nk - nq
  __device__ int q0() const { return 0; }  // first token row (variable-length layout)
  __device__ int k0() const { return 0; }
  __device__ int h() const { return 0; }
};

struct SeqVar {
  int nq_, nk_, nqt_, nkt_, q0_, k0_, h_;
  __device__ int nq() const { return nq_; }
  __device__ int nk() const { return nk_; }
  __device__ int nqt() const { return nqt_; }
  __device__ int nkt() const { return nkt_; }
  __device__ int causal_off() const { return nk_ - nq_; }
  __device__ int q0() const { return q0_; }
  __device__ int k0() const { return k0_; }
  __device__ int h() const { return h_; }
};

template <bool kVarlen>
__device__ __forceinline__ auto seq_of(const KernelParams& p, int bh) {
  if constexpr (!kVarlen) {
    return SeqDense{p};
  } else {
    const int b = bh / p.heads;
    const int qa = min(max(__ldg(p.cu_q + b), 0), p.total_q);
    const int qb = min(max(__ldg(p.cu_q + b + 1), qa), p.total_q);
    const int ka = min(max(__ldg(p.cu_k + b), 0), p.total_k);
    const int kb = min(max(__ldg(p.cu_k + b + 1), ka), p.total_k);
    SeqVar s;
    s.h_ = bh - b * p.heads;
    s.q0_ = qa;
    s.k0_ = ka;
    s.nq_ = qb - qa;
    s.nk_ = kb - ka;
    s.nqt_ = (s.nq_ + kBM - 1) / kBM;
    s.nkt_ = (s.nk_ + kBN - 1) / kBN;
    return s;
  }
}

// TMA coordinates (y, z) of a 128-row tile starting at sequence row `row`:
// dense maps are {D, N, B*H}, variable-length maps {D, H, T}.
template <bool kVarlen>
__device__ __forceinline__ void tile_coords(int row, int bh, int h, int tok0, int& y, int& z) {
  if constexpr (kVarlen) {
    y = h;
    z = tok0 + row;
  } else {
    y = row;
    z = bh;
  }
}

template <int D_, bool kFp8_ = false>
struct Cfg {
  static constexpr int kD = D_;
  static constexpr bool kFp8 = kFp8_;  // e4m3 Q, K, V (kind::f8f6f4); bf16 otherwise
  static_assert(D_ == 64 || D_ == 128, "head dim 64 or 128");
  static_assert(!kFp8_ || D_ == 128, "8-bit inputs: head dim 128 (one 128-byte swizzle row)");
  static constexpr int kEltBytes = kFp8_ ? 1 : 2;
  static constexpr int kBoxCols = 128 / kEltBytes;          // elements per 128-byte box row
  static constexpr int kBoxes = D_ * kEltBytes / 128;       // TMA boxes per tile
  static constexpr int kBoxBytes = 128 * 128;               // 128 rows x 128 B
  static constexpr int kTileBytes = 128 * D_ * kEltBytes;
  static constexpr int kKStep = kFp8_ ? 32 : 16;            // K of one MMA instruction
  static constexpr int kStages = (kTileBytes == 32768) ? 4 : 8;  // K/V ring slots
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  // q_full, q_empty, full[S], empty[S], s_full[2], p_full[2], o_full[2], o_empty[2],
  // p_half[2], s_free[2], pv_done[2], mma_done
  static constexpr int kNumBars = 2 + 2 * kStages + 15;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  // Tensor memory columns.  At d = 128, S_0, S_1, O_0, O_1 fill all 512 and P_q
  // is written over S_q (bf16: 64 columns, e4m3: 32).  At d = 64 there is room
  // for P_q of its own, so the next S_q can be computed while the softmax of
  // the current one still runs.
  static constexpr bool kSeparateP = (D_ == 64);
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO0 = 256;
  static constexpr uint32_t kTmemO1 = kSeparateP ? 320 : 384;
  static constexpr uint32_t kTmemP0 = kSeparateP ? 384 : kTmemS0;
  static constexpr uint32_t kTmemP1 = kSeparateP ? 448 : kTmemS1;
  // Online-softmax reference: the reference max moves when the running max
  // exceeds it by more than kRescale (log2 units), and P = 2^(x - m_ref +
  // kPShift).  bf16 P: shift 0, P <= 2^8.  e4m3 P: the exponent range is
  // narrow (normal from 2^-6, largest 448), so the reference moves sooner and
  // P is shifted up by 2^4: P <= 2^8 still, while values down to 2^-18 of the
  // reference survive the rounding.
  static constexpr float kRescale = kFp8_ ? 4.0f : 8.0f;
  static constexpr float kPShift = kFp8_ ? 4.0f : 0.0f;
  // One pair in kPolyEvery of each row's exp2 goes through exp2_poly2 on the
  // FMA pipe, the rest through MUFU.  Measured on B200 (A/B on one GPU):
  // bf16 runs best at 1 in 8 (+0.6 to +2.2 % over 1 in 4; 1 in 3 or more, or
  // none at all, is slower); e4m3, whose MMAs take half the time and leave
  // the softmax more MUFU-bound, at 1 in 4 (1 in 8 is 3 % slower there).
  static constexpr int kPolyEvery = kFp8_ ? 4 : 8;
};

// Dynamic shared memory of fa_fwd_kernel<C, kVarlen>: the tiles and barriers
// of C and, for variable-length batches, the first-unit table of up to
// kMaxVarlenSeqs sequences with the per-warp totals of its scan.
template <class C, bool kVarlen>
constexpr int fwd_smem_bytes() {
  return C::kSmemBytes + (kVarlen ? 4 * (kMaxVarlenSeqs + 1 + kThreads / 32) : 0);
}

// 2^x on the FMA pipe for two lanes (relieves the MUFU exp2 unit, which at
// head dim 128 would otherwise run exactly as fast as the tensor cores eat
// scores).  Cody-Waite range reduction x = n + f, n = round(x) via the
// 1.5 * 2^23 rounding constant, f in [-1/2, 1/2]; 2^f from a degree-3
// polynomial fitted for minimum relative error (max 7.6e-5, well under the
// bf16 rounding that follows; the fit is exact_attention_120_b200/exp2_poly_fit.py);
// 2^n added to the exponent field.  Arguments below -125 (masked scores are
// -inf) give 2^-125.  Arguments never exceed +8 here (see Cfg::kRescale).
// Cfg::kPolyEvery sets how many pairs take this path.
constexpr float kExp2Clamp = -125.0f;
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2C0 = 9.999282360e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426085174e-01f;
constexpr float kExp2C3 = 5.517049879e-02f;

__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, kExp2Clamp);
  x1 = fmaxf(x1, kExp2Clamp);
  float t0, t1, r0, r1, f0, f1, q0, q1;
  ptx::add2(t0, t1, x0, x1, kExp2Round, kExp2Round);    // n in the low mantissa bits
  ptx::add2(r0, r1, t0, t1, -kExp2Round, -kExp2Round);  // n as a float
  ptx::fma2(f0, f1, r0, r1, -1.f, -1.f, x0, x1);        // f = x - n
  ptx::fma2(q0, q1, f0, f1, kExp2C3, kExp2C3, kExp2C2, kExp2C2);
  ptx::fma2(q0, q1, q0, q1, f0, f1, kExp2C1, kExp2C1);
  ptx::fma2(q0, q1, q0, q1, f0, f1, kExp2C0, kExp2C0);
  y0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}


// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4)                           // D format: f32
         | (1u << 7)                         // A format: bf16
         | (1u << 10)                        // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)    // B major-ness
         | ((uint32_t)(N >> 3) << 17)        // N / 8
         | ((uint32_t)(M >> 4) << 24);       // M / 16
}

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format code 0), fp32
// accumulator, A K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool b_mn_major) {
  return (1u << 4)                           // D format: f32
         | ((b_mn_major ? 1u : 0u) << 16)    // B major-ness
         | ((uint32_t)(N >> 3) << 17)        // N / 8
         | ((uint32_t)(M >> 4) << 24);       // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
// lbo/sbo in bytes.  K-major tiles: sbo = 1024 (8 rows x 128 B), lbo unused.
// MN-major tiles: lbo = distance between 64-element column blocks, sbo = 1024.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Work unit taken by this CTA in its k-th round.  The units of round k are
// [k G, (k + 1) G) (G = gridDim.x), dealt to the CTAs forwards in even rounds
// and backwards in odd ones (`snake`): with the causal order (longest units
// first) a CTA that got one of the longest units of a round gets one of the
// shortest of the next, which balances the CTAs' total work (mid-size causal
// problems: +17 % measured).  Without `snake`, CTA c takes c, c + G, ...
// (variable-length batches, whose units have no such order: 6 % faster so).
// Increasing in k.
template <bool kSnake = true>
__device__ __forceinline__ int unit_of_round(int k) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
  return (kSnake && (k & 1)) ? (k + 1) * g - 1 - c : k * g + c;
}

__device__ __forceinline__ void decode_item(const KernelParams& p, int w, int& bh, int& pair,
                                            int& split) {
  split = w % p.splits;  // the slices of one unit run side by side
  w /= p.splits;
  if (p.causal) {
    // Longest rows first, heads interleaved within groups of p.group heads
    // whose K/V fit in L2 together (one group when all heads fit).
    const int per_group = p.group * p.npairs;
    const int g = w / per_group;
    const int r = w - g * per_group;
    const int gsz = min(p.group, p.bh - g * p.group);
    pair = p.npairs - 1 - r / gsz;
    bh = g * p.group + r % gsz;
  } else {  // all pairs of one head together: that head's K/V stays in L2
    bh = w / p.npairs;
    pair = w % p.npairs;
  }
}

// Query rows of sequence b of a variable-length batch, from the offsets
// clamped as in seq_of.
__device__ __forceinline__ int varlen_rows(const KernelParams& p, int b) {
  const int qa = min(max(__ldg(p.cu_q + b), 0), p.total_q);
  const int qb = min(max(__ldg(p.cu_q + b + 1), qa), p.total_q);
  return qb - qa;
}

// Work units of sequence b: one per pair of query tiles, for each head.
__device__ __forceinline__ int varlen_units(const KernelParams& p, int b) {
  const int nqt = (varlen_rows(p, b) + kBM - 1) / kBM;
  return p.heads * ((nqt + 1) >> 1);
}

// Variable-length batches deal only the units that exist: start[b] is the
// first unit of sequence b and start[nseq] their number, so sequences shorter
// than the longest leave no empty units behind (CTAs that skipped through
// empty units ran ahead of the others, and the K/V in use at once outgrew
// L2).  Whole block, ends with __syncthreads; start holds nseq + 1 entries
// followed by kThreads / 32 of scratch.
__device__ inline void build_unit_table(const KernelParams& p, int* start) {
  const int n = p.nseq;
  const int per = (n + kThreads - 1) / kThreads;
  const int b0 = min(n, (int)threadIdx.x * per), b1 = min(n, b0 + per);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += varlen_units(p, b);
  // Exclusive scan of the per-thread sums: within each warp, then across.
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int* warp_total = start + n + 1;
  if (lane == 31) warp_total[wid] = incl;
  __syncthreads();
  int run = incl - sum;
  for (int i = 0; i < wid; ++i) run += warp_total[i];
  for (int b = b0; b < b1; ++b) {
    start[b] = run;
    run += varlen_units(p, b);
  }
  if (threadIdx.x == kThreads - 1) start[n] = run;  // the last thread's run is the total
  __syncthreads();
}

// Unit w (< start[nseq]) of a variable-length batch.  The units of one
// sequence are consecutive; under the causal rule they run longest first with
// the heads interleaved in groups whose K/V fit in L2 together (group_keys
// keys per head), otherwise head by head.
__device__ __forceinline__ void decode_varlen(const KernelParams& p, const int* start, int w, int& bh,
                                              int& pair) {
  int lo = 0, hi = p.nseq - 1;  // the last sequence whose first unit is <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= w) lo = mid;
    else hi = mid - 1;
  }
  const int b = lo, r = w - start[b];
  const int np = (start[b + 1] - start[b]) / p.heads;  // units per head
  int h;
  if (p.causal) {
    const int ka = min(max(__ldg(p.cu_k + b), 0), p.total_k);
    const int nk = min(max(__ldg(p.cu_k + b + 1), ka), p.total_k) - ka;
    const int gs = nk > 0 ? min(p.heads, max(1, p.group_keys / nk)) : p.heads;
    const int g = r / (gs * np);
    const int rr = r - g * gs * np;
    const int gsz = min(gs, p.heads - g * gs);
    pair = np - 1 - rr / gsz;
    h = g * gs + rr % gsz;
  } else {
    h = r / np;
    pair = r - h * np;
  }
  bh = b * p.heads + h;
}

// Unit w of this launch: (b * H + h, pair of query tiles, key slice).
template <bool kVarlen>
__device__ __forceinline__ void decode_unit(const KernelParams& p, const int* start, int w, int& bh, int& pair,
                                            int& split) {
  if constexpr (kVarlen) {
    decode_varlen(p, start, w, bh, pair);
    split = 0;
  } else {
    decode_item(p, w, bh, pair, split);
  }
}

// Largest key index query tile qt can see under the causal rule (may be < 0).
template <class Seq>
__device__ __forceinline__ int causal_last_key(const Seq& sq, int qt) {
  return min(qt * kBM + kBM - 1, sq.nq() - 1) + sq.causal_off();
}

// Number of key tiles to scan for query tile qt: all of them, or under the
// causal rule those up to the tile of its last visible key.
template <class Seq>
__device__ __forceinline__ int key_tile_end(const KernelParams& p, const Seq& sq, int qt) {
  if (!p.causal) return sq.nkt();
  const int last = causal_last_key(sq, qt);
  return last < 0 ? 0 : min(sq.nkt(), last / kBN + 1);
}

// Bit l set <=> key tile j0 + l, which must lie in [jlo, jhi), is visible to
// query tile qt (whole warp calls).  The block mask (dense batches only) is
// indexed with the kernel-wide tile counts.
template <class Seq>
__device__ __forceinline__ uint32_t keep_bits(const KernelParams& p, const Seq& sq, int bh, int qt,
                                              int j0, int lane, int jlo, int jhi) {
  const int j = j0 + lane;
  bool k = (qt < sq.nqt()) && (j >= jlo) && (j < jhi);
  if (k && p.causal) k = j * kBN <= causal_last_key(sq, qt);
  if (k && p.mask != nullptr) k = p.mask[((size_t)bh * p.nqt + qt) * p.nkt + j] != 0;
  return __ballot_sync(0xffffffffu, k);
}

// Bounded wait for the phase of `bar` with parity `parity`.  Returns false if
// this wait timed out or, when `honor_abort`, the CTA is aborting because
// another role timed out.  Drain waits pass honor_abort = false: they must see
// their copies land (or time out) even while aborting.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      const KernelParams& p, bool honor_abort = true) {
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

// Whole-warp bounded wait: every lane polls, the result is warp-uniform.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          const KernelParams& p) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, p));
}

// Barrier addresses shared by the kernel and the MMA helpers.  Layout from
// bar0: q_full, q_empty, full[S], empty[S], s_full[2], p_full[2], o_full[2],
// o_empty[2], p_half[2], mma_done.
template <class C> __device__ __forceinline__ uint32_t bar_full(uint32_t bar0, int s) { return bar0 + 16 + 8u * s; }
template <class C> __device__ __forceinline__ uint32_t bar_q(uint32_t bar0) { return bar0 + 16 + 16u * C::kStages; }
template <class C> __device__ __forceinline__ uint32_t bar_s_full(uint32_t bar0, int q) { return bar_q<C>(bar0) + 8u * q; }
template <class C> __device__ __forceinline__ uint32_t bar_p_full(uint32_t bar0, int q) { return bar_q<C>(bar0) + 16 + 8u * q; }
template <class C> __device__ __forceinline__ uint32_t bar_o_full(uint32_t bar0, int q) { return bar_q<C>(bar0) + 32 + 8u * q; }
template <class C> __device__ __forceinline__ uint32_t bar_o_empty(uint32_t bar0, int q) { return bar_q<C>(bar0) + 48 + 8u * q; }
// P of keys [0, 64) of the tile is in tensor memory (p_full: all 128 keys).
template <class C> __device__ __forceinline__ uint32_t bar_p_half(uint32_t bar0, int q) { return bar_q<C>(bar0) + 64 + 8u * q; }
// Separate-P layout only: the softmax has read S_q (s_free), the PV MMAs of
// slot q's latest P are complete (pv_done).
template <class C> __device__ __forceinline__ uint32_t bar_s_free(uint32_t bar0, int q) { return bar_q<C>(bar0) + 80 + 8u * q; }
template <class C> __device__ __forceinline__ uint32_t bar_pv_done(uint32_t bar0, int q) { return bar_q<C>(bar0) + 96 + 8u * q; }
template <class C> __device__ __forceinline__ uint32_t bar_mma_done(uint32_t bar0) { return bar_q<C>(bar0) + 112; }

// The MMA of the configuration's kind (kind::f16 for bf16, kind::f8f6f4 for e4m3).
template <class C>
__device__ __forceinline__ void mma_ss_any(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (C::kFp8) ptx::mma_ss_f8(d, a, b, idesc, acc);
  else ptx::mma_ss(d, a, b, idesc, acc);
}
template <class C>
__device__ __forceinline__ void mma_ts_any(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (C::kFp8) ptx::mma_ts_f8(d, a, b, idesc, acc);
  else ptx::mma_ts(d, a, b, idesc, acc);
}

// MMA-issuer state of one query slot.
struct MmaSlot {
  int64_t pend = -1;     // ring index of the V tile owed a PV MMA, or -1
  uint32_t npv = 0;      // PV MMAs issued in this work unit
  uint32_t pwait = 0;    // p_full phases consumed
  uint32_t nitems = 0;   // work units seen with this slot valid
  uint32_t ns = 0;       // S MMAs issued (separate-P layout: s_free phases owed)
  bool need_oe = false;  // must wait for the previous unit's epilogue first
  __device__ __forceinline__ void begin_unit(bool valid) {
    pend = -1;
    npv = 0;
    need_oe = valid && nitems > 0;
  }
  __device__ __forceinline__ void end_unit(bool valid) {
    if (valid) ++nitems;
  }
};

template <class C>
struct MmaCtx {
  uint32_t tmem, sQ, sRing;
  volatile int* abort_flag;
};

// O_q += P_q V for the pending V of slot Q.  Called by the whole MMA warp
// (warp-uniform); one elected lane issues.
template <class C, int Q>
__device__ __forceinline__ bool mma_issue_pv(const MmaCtx<C>& c, const KernelParams& p, MmaSlot& s,
                                             int64_t& v_ready, uint32_t bar0) {
  constexpr int D = C::kD;
  constexpr uint32_t kIdescPV = C::kFp8 ? idesc_e4m3(128, D, true) : idesc_bf16(128, D, true);
  // One MMA per kKStep keys: A = 8 tensor-memory columns of P (32 bytes per
  // row), B = kKStep rows of V (MN-major, 128 B per row).
  constexpr int kSteps = kBN / C::kKStep;
  constexpr uint32_t kVStep = C::kKStep * 128;
  // Keys [0, 64) of P first: their MMAs overlap the softmax of keys [64, 128).
  if (!wait_warp(bar_p_half<C>(bar0, Q), s.pwait & 1u, c.abort_flag, p)) return false;
  ptx::tc_fence_after();
  const int64_t vr = s.pend;
  if (vr > v_ready) {
    if (!wait_warp(bar_full<C>(bar0, (int)(vr % C::kStages)), (uint32_t)(vr / C::kStages) & 1u,
                   c.abort_flag, p))
      return false;
    v_ready = vr;
    ptx::tc_fence_after();
  }
  if (s.need_oe) {  // the previous unit's epilogue has read O_q
    if (!wait_warp(bar_o_empty<C>(bar0, Q), (s.nitems - 1) & 1u, c.abort_flag, p)) return false;
    s.need_oe = false;
    ptx::tc_fence_after();
  }
  const uint32_t vbase = c.sRing + (uint32_t)(vr % C::kStages) * C::kTileBytes;
  const uint32_t tO = c.tmem + (Q ? C::kTmemO1 : C::kTmemO0);
  const uint32_t tP = c.tmem + (Q ? C::kTmemP1 : C::kTmemP0);
  const uint32_t acc0 = s.npv > 0 ? 1u : 0u;
#pragma unroll
  for (int kk = 0; kk < kSteps / 2; ++kk)
    if (ptx::elect_one())
      mma_ts_any<C>(tO, tP + kk * 8, smem_desc_sw128(vbase + kk * kVStep, C::kBoxBytes, 1024), kIdescPV,
                    kk > 0 ? 1u : acc0);
  if (!wait_warp(bar_p_full<C>(bar0, Q), s.pwait & 1u, c.abort_flag, p)) return false;
  ++s.pwait;
  ptx::tc_fence_after();
#pragma unroll
  for (int kk = kSteps / 2; kk < kSteps; ++kk)
    if (ptx::elect_one())
      mma_ts_any<C>(tO, tP + kk * 8, smem_desc_sw128(vbase + kk * kVStep, C::kBoxBytes, 1024), kIdescPV,
                    1u);
  if (C::kSeparateP && ptx::elect_one()) ptx::mma_commit(bar_pv_done<C>(bar0, Q));
  ++s.npv;
  s.pend = -1;
  return true;
}

// S_q = Q_q K_j^T into slot Q's S columns (warp-uniform).  With the
// separate-P layout the softmax must first have read the previous S_q.
template <class C, int Q>
__device__ __forceinline__ bool mma_issue_s(const MmaCtx<C>& c, const KernelParams& p, MmaSlot& s,
                                            int kslot, uint32_t bar0) {
  constexpr int D = C::kD;
  constexpr uint32_t kIdescQK = C::kFp8 ? idesc_e4m3(128, 128, false) : idesc_bf16(128, 128, false);
  if (C::kSeparateP && s.ns > 0) {
    if (!wait_warp(bar_s_free<C>(bar0, Q), (s.ns - 1) & 1u, c.abort_flag, p)) return false;
    ptx::tc_fence_after();
  }
  const uint32_t qbase = c.sQ + Q * C::kTileBytes;
  const uint32_t kbase = c.sRing + kslot * C::kTileBytes;
  const uint32_t tS = c.tmem + (Q ? C::kTmemS1 : C::kTmemS0);
  // Four K steps of 32 bytes per 128-byte box row.
#pragma unroll
  for (int kk = 0; kk < D / C::kKStep; ++kk) {
    const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
    if (ptx::elect_one())
      mma_ss_any<C>(tS, smem_desc_sw128(qbase + off, 16, 1024), smem_desc_sw128(kbase + off, 16, 1024),
                    kIdescQK, kk > 0 ? 1u : 0u);
  }
  if (ptx::elect_one()) ptx::mma_commit(bar_s_full<C>(bar0, Q));
  ++s.ns;
  return true;
}

// One kept K tile for slot Q in the P-over-S layout: settle its pending PV
// (P_q shares columns with S_q), then S_q = Q_q K_j^T.  Warp-uniform.
template <class C, int Q>
__device__ __forceinline__ bool mma_slot_step(const MmaCtx<C>& c, const KernelParams& p, MmaSlot& s,
                                              int64_t& v_ready, int kslot, uint32_t vr, uint32_t bar0) {
  if (s.pend >= 0 && !mma_issue_pv<C, Q>(c, p, s, v_ready, bar0)) return false;
  if (!mma_issue_s<C, Q>(c, p, s, kslot, bar0)) return false;
  s.pend = vr;
  return true;
}

template <class C, bool kVarlen = false>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_kernel(const __grid_constant__ KernelParams p) {
  constexpr int D = C::kD;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);

  const uint32_t sQ = base + C::kOffQ;
  const uint32_t sRing = base + C::kOffRing;
  const uint32_t bar0 = base + C::kOffBar;
  const uint32_t bQFull = bar0, bQEmpty = bar0 + 8;
  auto bFull = [&](int s) { return bar_full<C>(bar0, s); };
  auto bEmpty = [&](int s) { return bar0 + 16 + 8u * (C::kStages + s); };
  auto bSFull = [&](int q) { return bar_s_full<C>(bar0, q); };
  auto bPFull = [&](int q) { return bar_p_full<C>(bar0, q); };
  auto bOFull = [&](int q) { return bar_o_full<C>(bar0, q); };
  auto bOEmpty = [&](int q) { return bar_o_empty<C>(bar0, q); };
  auto bPHalf = [&](int q) { return bar_p_half<C>(bar0, q); };
  const uint32_t bMmaDone = bar_mma_done<C>(bar0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // The next attention launch on the stream may start its prologue now.
  ptx::launch_dependents();
  if (threadIdx.x == 0) {
    ptx::mbar_init(bQFull, 1);
    ptx::mbar_init(bQEmpty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(bFull(s), 1);
      ptx::mbar_init(bEmpty(s), 1);
    }
    for (int q = 0; q < 2; ++q) {
      ptx::mbar_init(bSFull(q), 1);
      ptx::mbar_init(bPFull(q), 128);
      ptx::mbar_init(bOFull(q), 1);
      ptx::mbar_init(bOEmpty(q), 128);
      ptx::mbar_init(bPHalf(q), 128);
      ptx::mbar_init(bar_s_free<C>(bar0, q), 128);
      ptx::mbar_init(bar_pv_done<C>(bar0, q), 1);
    }
    ptx::mbar_init(bMmaDone, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == kLoadWarp && lane == 0) {
    ptx::prefetch_tensormap(&p.tm_q);
    ptx::prefetch_tensormap(&p.tm_k);
    ptx::prefetch_tensormap(&p.tm_v);
  }
  if (warp == kMmaWarp) {
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
  int* unit_start = reinterpret_cast<int*>(base_ptr + C::kOffMisc + 16);
  int items = p.items;
  if constexpr (kVarlen) {
    build_unit_table(p, unit_start);
    items = unit_start[p.nseq];
  }

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ TMA producer ---
    uint32_t it = 0;       // K/V ring loads issued
    uint32_t nq = 0;       // Q loads issued
    bool ok = true;
    for (int k = 0, w = unit_of_round<!kVarlen>(0); w < items && ok && !p.starve_producer;
         w = unit_of_round<!kVarlen>(++k)) {
      int bh, pair, split;
      decode_unit<kVarlen>(p, unit_start, w, bh, pair, split);
      const auto sq = seq_of<kVarlen>(p, bh);
      const int qt0 = 2 * pair, qt1 = qt0 + 1;
      const int nvalid = (qt1 < sq.nqt()) ? 2 : 1;
      const int jb = split * p.kt_per_split, je = min(sq.nkt(), jb + p.kt_per_split);
      ok = wait_warp(bQEmpty, (nq & 1u) ^ 1u, abort_flag, p);
      if (ok && ptx::elect_one()) {
        ptx::mbar_arrive_expect_tx(bQFull, nvalid * C::kTileBytes);
        for (int q = 0; q < nvalid; ++q) {
          int y, z;
          tile_coords<kVarlen>((qt0 + q) * kBM, bh, sq.h(), sq.q0(), y, z);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            ptx::tma_load_3d(sQ + q * C::kTileBytes + bx * C::kBoxBytes, &p.tm_q, bQFull, bx * C::kBoxCols, y, z);
        }
      }
      ++nq;
      const int jend = min(je, key_tile_end(p, sq, qt0 + nvalid - 1));
      for (int j0 = jb & ~31; j0 < jend && ok; j0 += 32) {
        uint32_t u = keep_bits(p, sq, bh, qt0, j0, lane, jb, je) | keep_bits(p, sq, bh, qt1, j0, lane, jb, je);
        while (u != 0 && ok) {
          const int j = j0 + __ffs(u) - 1;
          u &= u - 1;
#pragma unroll
          for (int t = 0; t < 2; ++t) {  // K_j then V_j
            const int slot = it % C::kStages;
            ok = ok && wait_warp(bEmpty(slot), ((it / C::kStages) & 1u) ^ 1u, abort_flag, p);
            if (ok) {
              if (ptx::elect_one()) {
                ptx::mbar_arrive_expect_tx(bFull(slot), C::kTileBytes);
                const CUtensorMap* map = t == 0 ? &p.tm_k : &p.tm_v;
                int y, z;
                tile_coords<kVarlen>(j * kBN, bh, sq.h(), sq.k0(), y, z);
                for (int bx = 0; bx < C::kBoxes; ++bx)
                  ptx::tma_load_3d(sRing + slot * C::kTileBytes + bx * C::kBoxBytes, map,
                                   bFull(slot), bx * C::kBoxCols, y, z);
              }
              ++it;
            }
          }
        }
      }
    }
    // Drain: every load issued must have landed before the CTA may exit.
    const uint32_t first = it > (uint32_t)C::kStages ? it - C::kStages : 0u;
    for (uint32_t r = first; r < it; ++r)
      wait_bar(bFull(r % C::kStages), (r / C::kStages) & 1u, abort_flag, p, false);
    if (nq > 0) wait_bar(bQFull, (nq - 1) & 1u, abort_flag, p, false);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer ---
    MmaSlot slot0, slot1;         // per query slot state, kept in registers
    uint32_t it = 0;              // ring slots consumed (mirrors the producer)
    uint32_t nq = 0;              // Q tiles consumed
    int64_t v_ready = -1;         // ring index of the newest V whose load was awaited
    bool ok = true;
    const MmaCtx<C> ctx{tmem, sQ, sRing, abort_flag};
    for (int k = 0, w = unit_of_round<!kVarlen>(0); w < items && ok; w = unit_of_round<!kVarlen>(++k)) {
      int bh, pair, split;
      decode_unit<kVarlen>(p, unit_start, w, bh, pair, split);
      const auto sq = seq_of<kVarlen>(p, bh);
      const int qt0 = 2 * pair, qt1 = qt0 + 1;
      const bool valid1 = qt1 < sq.nqt();
      const int jb = split * p.kt_per_split, je = min(sq.nkt(), jb + p.kt_per_split);
      slot0.begin_unit(true);
      slot1.begin_unit(valid1);
      int64_t prev_v = -1;
      ok = wait_warp(bQFull, nq & 1u, abort_flag, p);
      ptx::tc_fence_after();
      ++nq;
      const int jend = min(je, key_tile_end(p, sq, valid1 ? qt1 : qt0));
      for (int j0 = jb & ~31; j0 < jend && ok; j0 += 32) {
        const uint32_t k0 = keep_bits(p, sq, bh, qt0, j0, lane, jb, je);
        const uint32_t k1 = keep_bits(p, sq, bh, qt1, j0, lane, jb, je);
        uint32_t u = k0 | k1;
        while (u != 0 && ok) {
          const int l = __ffs(u) - 1;
          u &= u - 1;
          const uint32_t kr = it, vr = it + 1;
          it += 2;
          const int kslot = kr % C::kStages;
          ok = wait_warp(bFull(kslot), (kr / C::kStages) & 1u, abort_flag, p);
          ptx::tc_fence_after();
          const bool keep0 = ((k0 >> l) & 1u) != 0, keep1 = ((k1 >> l) & 1u) != 0;
          if constexpr (C::kSeparateP) {
            // Both S first (the softmax has already read the previous S), then
            // the PVs of the previous tile, whose P lives in its own columns.
            if (ok && keep0) ok = mma_issue_s<C, 0>(ctx, p, slot0, kslot, bar0);
            if (ok && keep1) ok = mma_issue_s<C, 1>(ctx, p, slot1, kslot, bar0);
            if (ok && ptx::elect_one()) ptx::mma_commit(bEmpty(kslot));  // K_j no longer needed
            if (ok && slot0.pend >= 0) ok = mma_issue_pv<C, 0>(ctx, p, slot0, v_ready, bar0);
            if (ok && slot1.pend >= 0) ok = mma_issue_pv<C, 1>(ctx, p, slot1, v_ready, bar0);
            if (keep0) slot0.pend = vr;
            if (keep1) slot1.pend = vr;
          } else {
            // Slot q: pending O_q += P_q V first (P_q shares columns with S_q),
            // then S_q = Q_q K_j^T.
            if (ok && keep0) ok = mma_slot_step<C, 0>(ctx, p, slot0, v_ready, kslot, vr, bar0);
            if (ok && keep1) ok = mma_slot_step<C, 1>(ctx, p, slot1, v_ready, kslot, vr, bar0);
            if (ok && ptx::elect_one()) ptx::mma_commit(bEmpty(kslot));  // K_j no longer needed
            // A slot that skips K_j still owes a PV on the previous V: issue it
            // now so that V can be released.
            if (ok && !keep0 && slot0.pend >= 0) ok = mma_issue_pv<C, 0>(ctx, p, slot0, v_ready, bar0);
            if (ok && !keep1 && slot1.pend >= 0) ok = mma_issue_pv<C, 1>(ctx, p, slot1, v_ready, bar0);
          }
          if (ok && prev_v >= 0 && ptx::elect_one())
            ptx::mma_commit(bEmpty((int)(prev_v % C::kStages)));
          prev_v = vr;
        }
      }
      if (ok) {
        // Every S MMA of this unit is issued: Q may be replaced once they finish.
        if (ptx::elect_one()) ptx::mma_commit(bQEmpty);
        if (slot0.pend >= 0) ok = mma_issue_pv<C, 0>(ctx, p, slot0, v_ready, bar0);
        if (ok && slot1.pend >= 0) ok = mma_issue_pv<C, 1>(ctx, p, slot1, v_ready, bar0);
        if (ok && prev_v >= 0 && ptx::elect_one())
          ptx::mma_commit(bEmpty((int)(prev_v % C::kStages)));
        if (ok && ptx::elect_one()) {
          if (slot0.npv > 0) ptx::mma_commit(bar_o_full<C>(bar0, 0));
          if (valid1 && slot1.npv > 0) ptx::mma_commit(bar_o_full<C>(bar0, 1));
        }
      }
      slot0.end_unit(true);
      slot1.end_unit(valid1);
    }
    // Drain: every MMA issued must be complete before tensor memory is freed.
    if (ptx::elect_one()) ptx::mma_commit(bMmaDone);
    __syncwarp();
    wait_bar(bMmaDone, 0, abort_flag, p, false);
    __syncwarp();
  } else if (warp >= kFirstSoftmaxWarp) {
    // ---------------------------------------------------------- softmax ---
    const int q = (warp - kFirstSoftmaxWarp) >> 2;  // query slot 0 or 1
    const int row_in_tile = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (q ? C::kTmemS1 : C::kTmemS0);
    const uint32_t tO = tmem + lane_base + (q ? C::kTmemO1 : C::kTmemO0);
    const uint32_t tP = tmem + lane_base + (q ? C::kTmemP1 : C::kTmemP0);
    const float sl = p.scale_log2;
    uint32_t swait = 0, owait = 0;
    bool ok = true;
    for (int k = 0, w = unit_of_round<!kVarlen>(0); w < items && ok; w = unit_of_round<!kVarlen>(++k)) {
      int bh, pair, split;
      decode_unit<kVarlen>(p, unit_start, w, bh, pair, split);
      const auto sq = seq_of<kVarlen>(p, bh);
      const int qt = 2 * pair + q;
      const int jb = split * p.kt_per_split, je = min(sq.nkt(), jb + p.kt_per_split);
      if (qt >= sq.nqt()) continue;
      const int row = qt * kBM + row_in_tile;  // query row within the head
      float m_ref = -INFINITY;  // reference max, in units of c * score
      float l = 0.f;            // sum of bf16-rounded 2^(c s - m_ref)
      int n = 0;                // tiles processed
      const int jend = min(je, key_tile_end(p, sq, qt));
      for (int j0 = jb & ~31; j0 < jend && ok; j0 += 32) {
        uint32_t kb = keep_bits(p, sq, bh, qt, j0, lane, jb, je);
        while (kb != 0 && ok) {
          const int j = j0 + __ffs(kb) - 1;
          kb &= kb - 1;
          ok = wait_warp(bSFull(q), swait & 1u, abort_flag, p);
          ++swait;
          if (!ok) break;
          ptx::tc_fence_after();
          uint32_t r[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + 32 * c, r[c]);
          ptx::tmem_wait_ld();
          if constexpr (C::kSeparateP) {  // S_q may now be overwritten by the next tile
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_s_free<C>(bar0, q));
          }
          float s[128];
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(r[c >> 5][c & 31]);
          // Mask: keys past the causal diagonal and past the end of the
          // sequence (lim = last visible column of this tile, may be < 0).
          int lim = 127;
          if (p.causal) lim = min(lim, row + sq.causal_off() - j * kBN);
          lim = min(lim, sq.nk() - j * kBN - 1);
          if (lim < 127) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > lim) s[c] = -INFINITY;
          }
          // Row max over the 128 scores: 8 chains of three-input max (half
          // the dependent depth of 4 chains: +1 % measured), s[0..15] seed
          // the chains, s[16..127] are folded in pairs.
          float mx[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) mx[t] = fmaxf(s[2 * t], s[2 * t + 1]);
#pragma unroll
          for (int c = 16; c < 128; c += 16) {
#pragma unroll
            for (int t = 0; t < 8; ++t) mx[t] = ptx::max3(mx[t], s[c + 2 * t], s[c + 2 * t + 1]);
          }
          const float tmax = fmaxf(ptx::max3(mx[0], mx[1], mx[2]), ptx::max3(ptx::max3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
          const float m_new = fmaxf(m_ref, tmax * sl);
          // Move the reference max only when the new one exceeds it by more than
          // 2^kRescale (always on the first visible tile: m_ref = -inf).
          const bool rescale = m_new > m_ref + C::kRescale;
          float alpha = 1.f;
          if (rescale) {
            alpha = ptx::ex2(m_ref - m_new);  // 0 when m_ref = -inf
            l *= alpha;
            m_ref = m_new;
          }
          const float neg_m = (m_ref == -INFINITY) ? 0.f : C::kPShift - m_ref;
          if constexpr (C::kSeparateP) {
            // P_q and O_q are still read / written by the previous tile's PV.
            if (swait >= 2) {
              ok = wait_warp(bar_pv_done<C>(bar0, q), (swait - 2) & 1u, abort_flag, p);
              if (!ok) break;
              ptx::tc_fence_after();
            }
          }
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
          // Keys [0, 64) then [64, 128): each half of P is stored and signalled
          // as soon as it exists, so the PV MMAs of the first half overlap the
          // exponentials of the second.
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // P of keys [64 half, 64 half + 64): 32 words of two bf16, or 16
            // words of four e4m3; l sums exactly the rounded values.
            uint32_t pk[C::kFp8 ? 16 : 32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int cc = 32 * half + c;
              float x0, x1, p0, p1;
              ptx::fma2(x0, x1, s[2 * cc], s[2 * cc + 1], sl, sl, neg_m, neg_m);
              if (cc % C::kPolyEvery == C::kPolyEvery - 1) {
                exp2_poly2(p0, p1, x0, x1);
              } else {
                p0 = ptx::ex2(x0);
                p1 = ptx::ex2(x1);
              }
              if constexpr (C::kFp8) {
                if (c & 1) {
                  const uint32_t w4 = ptx::pack_e4m3x4(s[2 * cc - 2], s[2 * cc - 1], p0, p1);
                  pk[c >> 1] = w4;
                  ptx::add_e4m3x4(ls[2 * ((c >> 1) & 1)], ls[2 * ((c >> 1) & 1) + 1], w4);
                } else {
                  s[2 * cc] = p0;  // held until the next pair completes the word
                  s[2 * cc + 1] = p1;
                }
              } else {
                const uint32_t w2 = ptx::pack_bf16x2(p0, p1);
                pk[c] = w2;
                ptx::add_bf16x2(ls[2 * (c & 1)], ls[2 * (c & 1) + 1], w2);
              }
            }
            if constexpr (C::kFp8) ptx::tmem_st16(tP + 16 * half, pk);
            else ptx::tmem_st32(tP + 32 * half, pk);
            if (half == 0) {
              // O holds earlier tiles: rescale it in place before any PV of this
              // tile.  tcgen05.ld/st are warp-collective, so the warp rescales
              // together (alpha = 1 for rows whose reference did not move).
              if (n > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                  uint32_t t[32];
                  ptx::tmem_ld32(tO + 32 * c, t);
                  ptx::tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                  ptx::tmem_st32(tO + 32 * c, t);
                }
              }
              ptx::tmem_wait_st();
              ptx::tc_fence_before();
              ptx::mbar_arrive(bPHalf(q));
            }
          }
          l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bPFull(q));
          ++n;
        }
      }
      if (!ok) break;
      // ------------------------------------------------------- epilogue ---
      if (n > 0) {
        ok = wait_warp(bOFull(q), owait & 1u, abort_flag, p);
        ++owait;
        if (!ok) break;
        ptx::tc_fence_after();
      }
      // A row whose reference max never left -inf saw no visible key (masked
      // scores only add 2^-125 through the FMA-pipe exp2): O = 0, lse = -inf.
      const bool seen = m_ref != -INFINITY && l > 0.f;
      const float inv = seen ? p.o_scale / l : 0.f;
      const float lse2 = m_ref - C::kPShift + log2f(l);  // log2 of the row's sum, scaled scores
      // Sizes again (not held in registers across the tile loop).
      const auto se = seq_of<kVarlen>(p, bh);
      const bool in_range = row < se.nq();
      if (p.splits > 1) {
        // Partial result of this key slice: normalised O (fp32) and its lse.
        const size_t prow = (size_t)split * p.bh * p.Nq + (size_t)bh * p.Nq + (in_range ? row : 0);
        float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t t[32];
          if (n > 0) {
            ptx::tmem_ld32(tO + 32 * c, t);
            ptx::tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) t[e] = 0u;
          }
          if (in_range) {
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst[c * 8 + v4] = make_float4(__uint_as_float(t[4 * v4]) * inv, __uint_as_float(t[4 * v4 + 1]) * inv,
                                            __uint_as_float(t[4 * v4 + 2]) * inv, __uint_as_float(t[4 * v4 + 3]) * inv);
          }
        }
        if (in_range)
          p.part_lse[prow] = seen ? lse2 * 0.69314718055994530942f : -INFINITY;
      } else {
      // O row and lse element of this query: [B*H][Nq] rows, or token-major
      // [T][H] rows with lse [H][T] for variable-length batches.
      const int r = in_range ? row : 0;
      const size_t orow_i = kVarlen ? (size_t)(se.q0() + r) * p.heads + se.h() : (size_t)bh * p.Nq + r;
      const size_t lse_i = kVarlen ? (size_t)se.h() * p.total_q + se.q0() + r : (size_t)bh * p.Nq + r;
      uint4* orow = reinterpret_cast<uint4*>(p.o + orow_i * D);
      // The whole O row in one tensor-memory round trip (the scores are dead
      // here, so the registers are free), then 32-byte stores when O is
      // 32-byte aligned.
      uint32_t t[D / 32][32];
      if (n > 0) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(tO + 32 * c, t[c]);
        ptx::tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) t[c][e] = 0u;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t pkd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pkd[e] = ptx::pack_bf16x2(__uint_as_float(t[c][2 * e]) * inv, __uint_as_float(t[c][2 * e + 1]) * inv);
        if (in_range) {
          if (p.o_v8) {
            ptx::st_global_v8(orow + c * 4, pkd);
            ptx::st_global_v8(orow + c * 4 + 2, pkd + 8);
          } else {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              orow[c * 4 + v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
          }
        }
      }
      if (in_range)
        p.lse[lse_i] = seen ? lse2 * 0.69314718055994530942f : -INFINITY;
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bOEmpty(q));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
