// Placeholder until the tensor-core attention kernel lands.
#include "kernels.cuh"
namespace dsa {
bool attn_tc_supported(int, int, int) { return false; }
size_t attn_tc_workspace(int32_t, int, int, int) { return 0; }
dsa_status_t launch_attn_tc(const Rows&, int32_t, int32_t, const uint16_t*, const uint16_t*,
                            const int32_t*, int, float, uint16_t*, float*, void*, size_t,
                            cudaStream_t) { return DSA_ERR_UNSUPPORTED; }
}
