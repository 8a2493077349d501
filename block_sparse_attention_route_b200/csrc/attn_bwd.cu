// attn_bwd.cu -- sparse flash-attention backward (placeholder until the kernels land).
#include "common.cuh"

namespace bsa {

struct BwdWs {
  size_t dq_acc, delta, total;
};
inline size_t bwd_align(size_t x) { return (x + 255) & ~size_t(255); }
BwdWs bwd_ws_layout(const Geo& g, int r) {
  (void)r;
  BwdWs w;
  w.dq_acc = 0;
  w.delta = bwd_align((size_t)g.B * g.H * g.NBq * g.BS * g.D * 4);
  w.total = w.delta + bwd_align((size_t)g.B * g.H * g.NBq * g.BS * 4);
  return w;
}
struct BwdPtrs {
  const void *q, *k, *v, *kc, *vc, *o, *dO;
  const float* lse;
  const int *idx, *cnt;
  void *dq, *dk, *dv;
  char* ws;
};
bsa_status_t run_bwd(const Geo&, int, const BwdPtrs&, const BwdWs&, int, cudaStream_t) {
  return BSA_ERR_UNSUPPORTED;
}

}  // namespace bsa
