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
  kHdrTickets = 16,   // decode merge tickets start here (not used by fwd/bwd)
};

struct FwdParams {
  int B, H, Hkv, L, T, G, npairs;
  int n_units;
  float scale_log2;   // scale * log2(e)
  float log2_tau;     // log2(tau); -inf when tau == 0
  void* O;            // [B, L, H, D] bf16
  float* LSE;         // [B, H, L]
  uint8_t* tile_mask; // [B, H, T, T] or null
  uint32_t* err;      // device error word
  uint32_t* sched;    // persistent scheduler counter (zeroed before launch)
  uint64_t budget_ns;
};

}  // namespace mala
