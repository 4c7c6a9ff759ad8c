// Tensor-core (tcgen05) sparse prefill attention -- placeholder until the kernel lands.
#include "bsa_common.cuh"

namespace bsa {

bool prefill_tc_supported(bsa_dtype dt, int d, int b, int q_block, int K, int Hq, int Hk) {
  (void)dt; (void)d; (void)b; (void)q_block; (void)K; (void)Hq; (void)Hk;
  return false;
}

bsa_status prefill_tc(const void*, const void*, const void*, int, int, int, int, int, int,
                      const int*, const int*, int, int, int, const float*, int, void*, float*,
                      int*, cudaStream_t) {
  return BSA_ERR_UNSUPPORTED;
}

}  // namespace bsa
