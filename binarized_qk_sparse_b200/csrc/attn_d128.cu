// attn_d128.cu -- the fused kernel's instantiations at head dim 128 (the
// BinaryAttention kernel benchmark's head dim), in a translation unit of their
// own so that they compile in parallel with had_lib.cu (head dim 64 and the
// host code).  Linked into the same library.
#include "launch.cuh"

namespace had {
HAD_DISPATCH_INST(, 128)
}  // namespace had
