// libdd: the whole library as one translation unit (the device error word and
// the kernels share it without relocatable device code).
#include "dd_api.cu"
#include "dd_verify.cu"
#include "dd_attention.cu"
#include "dd_attention_tc.cu"
#include "dd_attention_tc2.cu"
#include "dd_select.cu"
#include "dd_static.cu"
