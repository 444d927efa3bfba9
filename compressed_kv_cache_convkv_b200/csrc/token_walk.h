// Launch shape shared by the per-frame streaming kernels.
#pragma once

namespace ckv {

// Token-walk launch shape of the per-frame streaming kernels (amax, e4m3 quantisation,
// dequantisation, key rotation): the `cols` = H * D/8 (head, 8-channel chunk) columns
// of a token are split into slabs of kTokenThreads; CTA x = walker * slabs + slab owns
// one column per thread and walks the frame's tokens walker, walker + walkers, ...;
// y and z index frames and K|V.  token_grid_x returns slabs * walkers.
constexpr int kTokenThreads = 128;
int token_grid_x(int T, int cols, int frames_yz);

}  // namespace ckv
