// Host/device parameter blocks and small shared definitions of the MALA kernels.
#pragma once

#include <cstdint>

namespace mala {

constexpr int kTile = 128;           // B_q = B_k = 128 rows / keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kWorkspaceHeader = 256;  // counters + error word at the start of a workspace

// Layout of the workspace header (uint32 words).
enum HeaderWord : int {
  kHdrError = 0,      // device error word (0 = ok)
  kHdrSched0 = 1,     // persistent-scheduler counters
  kHdrSched1 = 2,
  kHdrSched2 = 3,
};

// Call statistics in the workspace header: three uint64 counters at this byte offset,
// zeroed at the start of every call (legal tiles tested, retained tiles, V tiles loaded
// by decode).  Fwd / bwd count one per (b, h, i, j) tile; decode one per (b, h, t).
constexpr int kStatsOffset = 128;

#ifdef __CUDACC__
__device__ __forceinline__ void stats_add(unsigned long long* stats, uint32_t legal,
                                          uint32_t retained, uint32_t v_loaded) {
  if (!stats) return;
  if (legal) atomicAdd(stats + 0, static_cast<unsigned long long>(legal));
  if (retained) atomicAdd(stats + 1, static_cast<unsigned long long>(retained));
  if (v_loaded) atomicAdd(stats + 2, static_cast<unsigned long long>(v_loaded));
}

// Debug margins: float max into a global buffer whose entries start as the all-ones bit
// pattern (written by the host before the launch).  Non-negative values are combined as
// signed integers and negative ones as unsigned integers, which both order IEEE floats
// correctly; the all-ones start value is below every float under both views, so the
// first arrival always wins.  -0 is folded into +0 first.
__device__ __forceinline__ void atomic_max_f32(float* addr, float v) {
  if (v == 0.f) v = 0.f;
  if (v >= 0.f)
    atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
  else
    atomicMin(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

// Warp-wide maximum (all 32 lanes must call).
__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
#endif

// One query block of one sequence of a packed (varlen) batch, in the order the
// persistent CTAs take them (heaviest first).
struct VarlenBlock {
  int qrow0, krow0;  // packed row of the sequence's first query / first key
  int L, off;        // the sequence's query rows and causal offset (key rows - L)
  int i;             // query block within the sequence
  int pad[3];
};

struct FwdParams {
  int B, H, Hkv, L, T, G, npairs;  // L, T: query rows and query blocks
  int Lk, Tk, off;    // key rows and key blocks; query row q sits at position off + q
  int Lrows;          // rows of Q / O per batch entry (L; the packed total for varlen)
  const VarlenBlock* vtab;  // varlen: one entry per (sequence, query block), else null
  int n_units;
  float scale_log2;   // scale * log2(e)
  float log2_tau;     // log2(tau); -inf when tau == 0
  void* O;            // [B, L, H, D] bf16
  float* LSE;         // [B, H, L]
  uint8_t* tile_mask; // [B, H, T, Tk] or null
  float* tile_margin; // [B, H, T, Tk] debug margins (natural log) or null
  uint32_t* err;      // device error word
  uint32_t* sched;    // persistent scheduler counter (zeroed before launch)
  uint64_t budget_ns;
  unsigned long long* stats;  // call statistics (kStatsOffset) or null
};

}  // namespace mala
