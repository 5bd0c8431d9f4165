// Tensor-core (tcgen05) attention: placeholder until the sm_100a kernel lands.
#include "kernels.h"
namespace thin {
bool attention_tc_supported(int, int, int) { return false; }
int attention_tc_tile_rows() { return 128; }
cudaError_t launch_attention_tc(const AttnArgs&, int*, cudaStream_t, bool* done) {
  *done = false;
  return cudaSuccess;
}
}  // namespace thin
