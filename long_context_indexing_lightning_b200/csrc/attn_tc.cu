// Sparse MLA attention on the tensor cores (placeholder until the tcgen05 kernel lands).
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
bool attn_tc_supported(int, int, int, int) { return false; }
size_t attn_workspace_bytes(int, int, int, int, int, int, int, int) { return 0; }
dsa_status_t attn_tc(const AttnArgs&) { return DSA_ERR_UNSUPPORTED; }
}  // namespace dsa
