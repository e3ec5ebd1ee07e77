// libcrs: the whole library as one translation unit (device globals such as the
// error word are shared by every kernel without relocatable device code).
#include "api.cu"
#include "lsh_tc.cu"
#include "lsh.cu"
#include "lsh_csr.cu"
#include "lsh_decode.cu"
#include "sparse_attn.cu"
#include "indexer.cu"
#include "indexer_tc.cu"
#include "blocks.cu"
#include "hisa.cu"
#include "route.cu"
#include "noalloc.cu"
