// Decode kernel instantiation for head_dim 128, 8 query heads per kv head.
#include "rq_decode.cuh"

RQ_DECODE_INSTANTIATE(128, 8)
