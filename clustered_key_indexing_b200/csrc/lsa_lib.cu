// lsa_lib.cu -- single translation unit of liblsa.so (one copy of the
// device-side error word, no separate device link step).
#include "lsa_build.cu"
#include "lsa_select.cu"
#include "lsa_attn.cu"
#include "lsa_band.cu"
#include "lsa_api.cu"
#include "lsa_decode.cu"
#include "lsa_noalloc.cu"
#include "lsa_pca.cu"
#include "lsa_probe.cu"
#include "lsa_bwd.cu"
#include "lsa_shard.cu"
