// Dion / Orth-Dion low-rank step (placeholder until its kernels land).
#include "internal.h"

extern "C" size_t dion_workspace_bytes(const ouo_mat* M, int nmat,
                                       const ouo_dion_params* p) {
  (void)M; (void)nmat; (void)p;
  return 0;
}

extern "C" int dion_lowrank_step(const ouo_mat* M, const ouo_mat* G,
                                 int g_dtype, const ouo_mat* Q_state,
                                 const ouo_mat* W, int w_dtype, int nmat,
                                 const ouo_dion_params* p, const float* scale,
                                 void* ws, size_t ws_bytes, int* dev_status,
                                 void* stream) {
  (void)M; (void)G; (void)g_dtype; (void)Q_state; (void)W; (void)w_dtype;
  (void)nmat; (void)p; (void)scale; (void)ws; (void)ws_bytes;
  (void)dev_status; (void)stream;
  return ouo::set_error(OUO_ERR_UNSUPPORTED, "dion_lowrank_step: not built yet");
}
