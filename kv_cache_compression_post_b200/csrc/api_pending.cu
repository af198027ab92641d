// Entry points whose kernels are not in this file set yet.
#include "bank.h"

extern "C" {
kvb_status kvb_forcing_init(kvb_bank*, cudaStream_t) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_forcing_export(kvb_bank*, int32_t, int32_t, int32_t*, void*, void*, int32_t*, cudaStream_t) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_prune_hybrid(kvb_bank*, int32_t, const uint8_t*, const void*, const void*, const void*, const int32_t*, int32_t, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_segment_cosine(const void*, const void*, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, kvb_dtype, float*, void*) { return KVB_E_UNSUPPORTED; }
}
