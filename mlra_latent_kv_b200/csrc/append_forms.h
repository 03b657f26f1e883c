// Which form latent_append takes for a shape (cache_kernels.cu).
#pragma once

namespace mlra {

// True when launch_append takes the two-kernel form, whose split-K partial
// sums need KS * B * (d_c + d_r) floats at its `part` argument (KS = ceil(D /
// 64)); false for the one-launch form, which keeps them on chip and leaves
// `part` unused.
bool append_uses_scratch(int dtype, int D, int d_c, int d_r);

}  // namespace mlra
