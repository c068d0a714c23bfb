// FMA split kernel variants for head_dim 128.
#include "split_variants.cuh"

namespace pda {
cudaError_t launch_split_d128(int kv, int mt, int tw, const SplitArgs& a, dim3 g,
                             cudaStream_t s) {
  return launch_for_dim<128>(kv, mt, tw, a, g, s);
}
}  // namespace pda
