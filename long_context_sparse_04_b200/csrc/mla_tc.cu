// mla_tc.cu - tensor-core sparse MLA (placeholder until the tcgen05 kernel lands).
#include "dsa_kernels.cuh"

namespace dsa {
bool mla_tc_supported(const MlaArgs&) { return false; }
int mla_tc_splits(int) { return 1; }
size_t mla_ws_bytes(int, int, int, int) { return 0; }
dsa_status launch_mla_tc(const MlaArgs&, cudaStream_t) { return DSA_ERR_UNSUPPORTED; }
}  // namespace dsa
