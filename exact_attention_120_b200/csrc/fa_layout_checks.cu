// Build-time checks of the kernels' resource layouts: every configuration's
// shared memory fits a CTA's 227 KB opt-in limit, every tensor-memory region
// lies inside the 512 columns one CTA allocates and regions that are live at
// the same time do not overlap, and TMA boxes and tiles keep the 1024-byte
// alignment the 128-byte swizzle needs.  Nothing here runs; a violated
// layout stops the build instead of corrupting memory at run time.

#include "fa_bwd_kernel.cuh"
#include "fa_fwd_kernel.cuh"

namespace fa {
namespace {

constexpr int kMaxSmemPerCta = 232448;  // 227 KB, sm_100 opt-in maximum

template <class C>
constexpr bool fwd_layout_ok() {
  constexpr uint32_t D = C::kD;
  // O_0, O_1 fp32 accumulators after S_0, S_1.
  static_assert(C::kTmemO0 >= C::kTmemS1 + 128, "O_0 overlaps S_1");
  static_assert(C::kTmemO1 >= C::kTmemO0 + D, "O_1 overlaps O_0");
  static_assert(C::kTmemO1 + D <= kTmemCols, "O_1 past the allocation");
  // P: over S (bf16 64 columns, e4m3 32) or in its own columns.
  constexpr uint32_t kPCols = C::kFp8 ? 32 : 64;
  if constexpr (C::kSeparateP) {
    static_assert(C::kTmemP0 >= C::kTmemO1 + D, "P_0 overlaps O_1");
    static_assert(C::kTmemP1 >= C::kTmemP0 + kPCols, "P_1 overlaps P_0");
    static_assert(C::kTmemP1 + kPCols <= kTmemCols, "P_1 past the allocation");
  } else {
    static_assert(C::kTmemP0 == C::kTmemS0 && C::kTmemP1 == C::kTmemS1, "P over S");
    static_assert(kPCols <= 128, "P wider than S");
  }
  static_assert(C::kSmemBytes <= kMaxSmemPerCta, "shared memory over the per-CTA limit");
  // Variable-length batches add the table of the sequences' first work units.
  static_assert(fwd_smem_bytes<C, true>() <= kMaxSmemPerCta, "variable-length table over the per-CTA limit");
  static_assert(C::kOffRing % 1024 == 0 && C::kTileBytes % 1024 == 0, "swizzle-atom alignment");
  static_assert(C::kBoxes * C::kBoxBytes == C::kTileBytes, "tile = whole TMA boxes");
  static_assert(C::kOffBar % 8 == 0, "mbarrier alignment");
  return true;
}

template <int D>
constexpr bool bwd_layout_ok() {
  using C = BwdCfg<D>;
  // Half-buffers [0, 256); dK/dV launch: dV, dK; dQ launch: dQ, Q, dO.
  static_assert(C::g_col(1) + 64 <= C::kAcc0, "half-buffers overlap the accumulators");
  static_assert(C::kAcc1 >= C::kAcc0 + D && C::kAcc1 + D <= kTmemCols, "dV / dK past the allocation");
  static_assert(C::kTq == C::kAcc0 + D, "Q right after dQ");
  static_assert(C::kTdo == C::kTq + D / 2 && C::kTdo + D / 2 <= kTmemCols, "dO past the allocation");
  static_assert(C::kSmemBytes <= kMaxSmemPerCta, "shared memory over the per-CTA limit");
  static_assert(C::kOffRing % 1024 == 0 && C::kTileBytes % 1024 == 0, "swizzle-atom alignment");
  static_assert(C::kOffBar % 8 == 0 && C::kOffVals % 16 == 0, "barrier / vector alignment");
  return true;
}

static_assert(fwd_layout_ok<Cfg<64>>() && fwd_layout_ok<Cfg<128>>() && fwd_layout_ok<Cfg<128, true>>(),
              "forward layouts");
static_assert(bwd_layout_ok<64>() && bwd_layout_ok<128>(), "backward layouts");

}  // namespace
}  // namespace fa
