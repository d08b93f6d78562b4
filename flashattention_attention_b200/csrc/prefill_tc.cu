// prefill_tc.cu -- tensor-core (tcgen05) prefill; under construction.
#include "internal.h"

namespace fa {
fa_status launch_prefill_tc(const fa_fwd_params& p, const LaunchCtx& ctx) {
  (void)p;
  (void)ctx;
  return FA_ERR_UNSUPPORTED;
}
}  // namespace fa
