// Single translation unit of libdvssq.so: the kernels share device state (the
// error word) and helpers without relocatable device code.
#include "dvssq_api.cu"
#include "fwht.cu"
#include "glue.cu"
#include "encode.cu"
#include "decode.cu"
#include "decode_row.cu"
#include "prefill.cu"
#include "stack.cu"
#include "materialize.cu"
#include "lowrank.cu"
#include "selftest.cu"
#include "static_scratch.cu"
