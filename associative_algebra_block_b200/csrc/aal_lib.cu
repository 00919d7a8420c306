// libaal is built as a single translation unit so that every kernel can reach
// the device status word without relocatable device code.
#include "aal_api.cu"
#include "aal_simt.cu"
#include "aal_decode.cu"
#include "aal_tc.cu"
#include "aal_ffn_decode.cu"
#include "aal_segments.cu"
#include "aal_fixed_scratch.cu"
