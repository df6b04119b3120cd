// gdla_lib.cu - the single translation unit libgdla.so is built from, so the
// device-side failure word is one symbol without relocatable device code.
#include "gdla_api.cu"
#include "gdla_prefill.cu"
#include "gdla_prefill_bwd.cu"
#include "gdla_prologue.cu"
#include "gdla_decode.cu"
#include "gdla_decode_noalloc.cu"
#include "gdla_decode_latent.cu"
#include "gdla_selftest.cu"
