// File-backed K/V store with a bounded page cache in host memory.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.2 (tiered KV
// storage): RAM-backed history, or a filesystem store in which RAM is a
// bounded page cache over disk (NVMe).  The host side (file IO, the page
// cache, its replacement policy) is in kv_store.cpp; the device gather that
// reads the cache is gather_store_kernel in tier.cuh.  This header holds the
// handle's layout, shared by the two translation units.
#pragma once
#include <stdint.h>

#include <string>
#include <vector>

#include "hga.h"

struct hga_kv_store {
  std::string path;
  int fd_write = -1;            // buffered descriptor for appends and plain reads
  int fd_read = -1;             // descriptor for page reads (O_DIRECT when asked)
  bool direct = false;

  // geometry
  int32_t dtype = 0;
  int64_t Hkv = 0, d = 0, elem = 0;
  int64_t t_cap = 0, page_tokens = 0, n_pages = 0;   // n_pages per KV head
  int64_t half_bytes = 0;       // page_tokens * d * elem: the K (or V) half of a page
  int64_t page_bytes = 0;       // 2 * half_bytes
  int64_t length = 0;           // tokens appended

  // page cache (caller memory)
  char* cache = nullptr;
  int64_t cache_pages = 0;
  int32_t* page_table = nullptr;            // [Hkv][n_pages] -> slot or -1
  std::vector<int64_t> slot_page;           // slot -> global page (h * n_pages + n), -1 free
  std::vector<int32_t> prev, next;          // LRU list over occupied slots
  int32_t lru_head = -1, lru_tail = -1;     // head = most recently used
  std::vector<int32_t> free_slots;
  std::vector<uint32_t> slot_step;          // step that last needed the slot
  std::vector<uint32_t> page_step;          // per global page: step that listed it
  uint32_t step = 0;
};
