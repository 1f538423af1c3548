// beacon_score_tc.cu -- tcgen05 (5th-generation tensor core) beacon score for
// bf16 caches.  Placeholder until the tensor-core kernel lands: reports
// "not supported" so the SIMT kernel serves every case.
#include "kvc_internal.h"

namespace kvc {

bool beacon_score_tc_supported(int d, int B, int dtype) {
  (void)d;
  (void)B;
  (void)dtype;
  return false;
}

cudaError_t launch_beacon_score_tc(const BeaconScoreParams &p, int n_req, int max_l,
                                   cudaStream_t s) {
  (void)p;
  (void)n_req;
  (void)max_l;
  (void)s;
  return cudaErrorNotSupported;
}

}  // namespace kvc
