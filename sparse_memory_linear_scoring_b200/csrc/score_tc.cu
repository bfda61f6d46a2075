// score_tc.cu -- tensor-core (tcgen05) sub-key scoring; filled in below.
#include "sdm_internal.cuh"

namespace sdm {

bool score_tc_supported(const sdm_dims* d) { (void)d; return false; }
int score_tc_capacity(const sdm_dims* d) { return d->k; }
size_t score_tc_smem(const Plan& p) { (void)p; return 0; }
cudaError_t launch_score_tc(const Plan& p, const void* q, const void* k, const void* C1,
                            const void* C2, int t0, int tlen, int* surv_cnt, uint2* surv,
                            int* redo_rows, DevStatus* st, cudaStream_t s) {
  (void)p; (void)q; (void)k; (void)C1; (void)C2; (void)t0; (void)tlen; (void)surv_cnt;
  (void)surv; (void)redo_rows; (void)st; (void)s;
  return cudaErrorNotSupported;
}

}  // namespace sdm
