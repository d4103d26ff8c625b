// dcp_mla.cu -- MLA (absorbed, shared 576-wide latent) partial decode attention.
#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {

int mla_ctas() { return device_sm_count(); }

dcp_status launch_mla_decode(const dcp_attn_desc&, int, const ShardSet&, const void*, const int32_t*, void*, size_t,
                             cudaStream_t) {
  return DCP_ERR_UNSUPPORTED;
}

}  // namespace dcp
