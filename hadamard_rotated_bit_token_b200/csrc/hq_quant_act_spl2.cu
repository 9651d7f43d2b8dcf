// hq_quant_act_spl2.cu -- the warp-row activation quantizer with 2 slices a
// lane (K = 2048), instantiated in its own translation unit (see hq_quant_act.cu).
#define HQ_ACT_PART 2
#include "hq_quant_act.cu"
