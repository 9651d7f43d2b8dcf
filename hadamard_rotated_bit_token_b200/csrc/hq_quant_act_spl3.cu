// hq_quant_act_spl3.cu -- the warp-row activation quantizer with 3 slices a
// lane (K = 3072), instantiated in its own translation unit (see hq_quant_act.cu).
#define HQ_ACT_PART 3
#include "hq_quant_act.cu"
