// hq_quant_act_spl4.cu -- the warp-row activation quantizer with 4 slices a
// lane (K = 4096), instantiated in its own translation unit (see hq_quant_act.cu).
#define HQ_ACT_PART 4
#include "hq_quant_act.cu"
