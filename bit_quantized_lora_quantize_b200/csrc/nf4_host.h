// Host-side construction of the NF4 levels and of the encoder's rounding
// boundaries.  Independent of any other implementation of the codebook: the
// normal quantile is found by Newton iteration on the C library's erfc.
#pragma once

#include "nf4_device.cuh"

namespace qlora {

// Levels: standard-normal quantiles at evenly spaced probabilities, 8 on the
// positive side and 7 on the negative side, plus an exact zero, divided by
// the largest one ("1. 4-bit NormalFloat (NF4)": every bucket gets an equal
// share of normally distributed values).  Outermost probability
// delta = 1 - (1/30 + 1/32)/2.  Computed in double, rounded once to float.
void nf4_levels(float out[16]);

// Levels plus, for j = 0..14, the exact boundary B_j in x / c at which the
// float32 quotient reaches the smallest float above the midpoint of levels
// j and j + 1.  Computed once per process; thread-safe.
const Nf4Params& nf4_params();

// The same for each 4-bit code of include/qlora.h (0 NF4, 1 FP4, 2 Int4):
// null for an unknown code; code_params falls back to NF4.
const Nf4Params* code_params_or_null(int code);
const Nf4Params& code_params(int code);

}  // namespace qlora
