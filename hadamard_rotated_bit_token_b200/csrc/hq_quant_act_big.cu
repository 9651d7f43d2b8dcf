// hq_quant_act_big.cu -- the segment activation quantizer for rows of more than
// 256 slices (K above 8192; up to 480 consumer threads, one CTA per SM),
// instantiated in its own translation unit (see hq_quant_act.cu).
#define HQ_ACT_PART 5
#include "hq_quant_act.cu"
