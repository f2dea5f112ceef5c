// Host-side construction of the NF4 level table and of the quantizer's bin table.
#pragma once
#include <stdint.h>

namespace qlora {

// One entry of the quantizer's bin table.  The normalised value xn in [-1, 1]
// falls in bin j = round_half_even(32 * xn) (-32..32), stored at index j mod 128.
// Each bin holds at most one decision threshold, so the code is  c + (xn > t)
// with t = +2 for a bin without a threshold.  The unused indices exist only so
// that a masked index computed from a non-finite value stays inside the table.
struct QuantBin {
  float t;
  int32_t c;
};
constexpr int kQuantBins = 128;

struct Nf4Tables {
  float levels[16];      // ascending, levels[0] = -1, levels[7] = 0, levels[15] = 1
  float thresholds[15];  // RD32((levels[i] + levels[i+1]) / 2)
  QuantBin bins[kQuantBins];
  float rcp[128];        // RN32(1 / (1 + k/128)), k = 0..127
  bool ok;               // construction invariants held
};

// Built once (thread-safe static); pure host arithmetic in double precision.
const Nf4Tables &nf4_tables();

}  // namespace qlora
