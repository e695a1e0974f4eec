// tq_lib.cu -- single translation unit of libtq.so (the device status word and the helpers are
// shared by every kernel without relocatable device code).
#include "tq_api.cu"
#include "tq_generic.cu"
#include "tq_pack.cu"
#include "tq_decode.cu"
#include "tq_batch.cu"
#include "tq_tcbatch.cu"
#include "tq_prefill.cu"
