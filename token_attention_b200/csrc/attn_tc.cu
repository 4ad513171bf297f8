// attn_tc.cu -- fused MTA attention on the sm_100a tensor cores (bf16).
#include "internal.h"

namespace mta {

bool attn_tc_supported(const AttnArgs &) { return false; }

cudaError_t launch_attn_tc(const AttnArgs &, const GnArgs *) { return cudaErrorNotSupported; }

}  // namespace mta
