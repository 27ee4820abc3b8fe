// Forward attention on the Blackwell tensor-memory path (tcgen05): placeholder
// until the kernel lands; fa_fwd falls back to the mma.sync kernel.
#include "fa_kernels.h"

namespace fa {

bool fwd_tc_supported(const FwdParams&) { return false; }

cudaError_t launch_fwd_tc(const FwdParams&, fa_dtype, cudaStream_t, int*) { return cudaErrorNotSupported; }

}  // namespace fa
