// Bank-level C entry points (placeholder until the admit pipeline lands).
#include "host_util.h"

extern "C" {
size_t kvb_workspace_size(const kvb_config*) { return 0; }
kvb_status kvb_bank_create(const kvb_config*, void*, size_t, void*, kvb_bank**) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_bank_destroy(kvb_bank*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_admit(kvb_bank*, int32_t, const void*, const void*, const int32_t*, int32_t, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_prune_hybrid(kvb_bank*, int32_t, const uint8_t*, const void*, const void*, const void*, const int32_t*, int32_t, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_attend(kvb_bank*, int32_t, const void*, int32_t, const void*, const void*, int32_t, const void*, const void*, int32_t, void*, float*, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_read_stats(kvb_bank*, int32_t, kvb_admit_stats*, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_bank_export(kvb_bank*, int32_t, int32_t, int32_t*, float*, float*, void*, void*, int32_t*, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_bank_import(kvb_bank*, int32_t, int32_t, const int32_t*, const float*, const float*, const void*, const void*, int32_t, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_device_status(kvb_bank*, void*) { return KVB_E_UNSUPPORTED; }
kvb_status kvb_segment_cosine(const void*, const void*, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, kvb_dtype, float*, void*) { return KVB_E_UNSUPPORTED; }
}
