// topk_narrow.cu -- the top-k selection in 256-thread CTAs at <= 64 registers,
// for the chunks of a prefill whose selection runs on a side stream while the
// next chunk's indexer runs (its CTAs take SMs as the indexer's retire).
#define DSA_TOPK_THREADS 256
#define DSA_TOPK_MIN_CTAS 4
#define DSA_TOPK_LAUNCH launch_topk_narrow
#include "topk_impl.cuh"
