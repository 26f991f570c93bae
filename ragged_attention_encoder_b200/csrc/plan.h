// Host-side plan builder: validation, work tiles, split-KV schedule, merge map.
// Pure C++ (no CUDA calls), so that it can be exercised on a machine without a GPU.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "rae.h"
#include "rae_internal.h"

namespace rae {

// Validates a configuration; returns RAE_OK or a status with a message.
int check_config(const rae_config& cfg, std::string* err);

// Upper bound on the CTAs any plan launches for cfg.
int32_t max_ctas_for(const rae_config& cfg);

// Size in int32 words of one plan image for cfg.
int64_t image_words_for(const rae_config& cfg);

// Builds a paged cross-attention plan image into `image` (image_words int32 words).
// causal: the queries of request b are the last qlen tokens of its kv_len-token sequence
// and query i sees keys [0, kv_len - qlen + i] (paged causal self-attention).
int build_paged_plan(const rae_config& cfg, const int32_t* qo_indptr,
                     const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                     const int32_t* kv_len, int32_t batch, int32_t num_pages, int32_t* image,
                     int64_t image_words, rae_plan* out, std::string* err, bool causal = false);

// Builds a ragged attention plan image.  cu_kv == nullptr means self-attention.
int build_ragged_plan(const rae_config& cfg, const int32_t* cu_q, const int32_t* cu_kv,
                      int32_t num_spans, int32_t block_size, int32_t* image, int64_t image_words,
                      rae_plan* out, std::string* err);

// One page's share of a K/V write: `ntok` tokens starting at packed source row `src_row` go
// to slots [slot0, slot0 + ntok) of page `page`.
struct WriteItem {
  int32_t src_row;
  int32_t ntok;
  int32_t page;
  int32_t slot0;
};

// Validates a K/V write and lists its page copies into `items` (capacity max_items).  The
// cu_src[b+1] - cu_src[b] tokens of request b go to sequence positions start[b], start[b]+1,
// ... of its pages (start == nullptr: from position 0, the context write).
int build_write_items(const rae_config& cfg, const int32_t* cu_src, const int32_t* page_indptr,
                      const int32_t* page_indices, const int32_t* start, int32_t batch,
                      int32_t num_pages, WriteItem* items, int64_t max_items, int64_t* num_items,
                      std::string* err);

}  // namespace rae
