// File-backed K/V store: the host side (file IO and the page cache).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.2 (tiered KV
// storage): the history may live in a filesystem store in which RAM is a
// bounded page cache over disk, suited to NVMe.  Here a page is page_tokens
// tokens of one KV head, K then V, in the file at (h * n_pages + n) *
// page_bytes.  Before a step's gather, hga_store_prepare lists the pages the
// step's history groups fall in (sink, routed, local window below t_hist),
// keeps the resident ones, and reads the rest into free or least recently
// used slots with a few threads issuing positional reads side by side (NVMe
// needs several requests in flight to reach its bandwidth).  The device never
// sees the file: gather_store_kernel copies from the cache slots, through the
// page table, into the device mirrors.
#include "kv_store.h"

#include <errno.h>
#include <fcntl.h>
#include <string.h>
#include <sys/stat.h>
#include <sys/uio.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <new>
#include <thread>

namespace {

constexpr int64_t kMaxRunPages = 256;           // iovecs per vectored read (<= IOV_MAX)

bool pread_full(int fd, char* dst, int64_t bytes, int64_t off) {
  while (bytes > 0) {
    ssize_t r = ::pread(fd, dst, (size_t)bytes, (off_t)off);
    if (r < 0) {
      if (errno == EINTR) continue;
      return false;
    }
    if (r == 0) {            // end of file: the rest was never written
      memset(dst, 0, (size_t)bytes);
      return true;
    }
    dst += r;
    off += r;
    bytes -= r;
  }
  return true;
}

// Reads one contiguous file range into scattered buffers (one run of
// adjacent pages into their cache slots); zero-fills past the end of file.
bool preadv_full(int fd, struct iovec* iov, int n, int64_t off) {
  int i = 0;
  while (i < n) {
    ssize_t r = ::preadv(fd, iov + i, n - i, (off_t)off);
    if (r < 0) {
      if (errno == EINTR) continue;
      return false;
    }
    if (r == 0) {
      for (; i < n; ++i) memset(iov[i].iov_base, 0, iov[i].iov_len);
      return true;
    }
    off += r;
    while (i < n && (size_t)r >= iov[i].iov_len) {
      r -= (ssize_t)iov[i].iov_len;
      ++i;
    }
    if (i < n && r > 0) {
      iov[i].iov_base = static_cast<char*>(iov[i].iov_base) + r;
      iov[i].iov_len -= (size_t)r;
    }
  }
  return true;
}

bool pwrite_full(int fd, const char* src, int64_t bytes, int64_t off) {
  while (bytes > 0) {
    ssize_t r = ::pwrite(fd, src, (size_t)bytes, (off_t)off);
    if (r < 0) {
      if (errno == EINTR) continue;
      return false;
    }
    src += r;
    off += r;
    bytes -= r;
  }
  return true;
}

bool same_layout(const hga_kv_store* s, const hga_params* p) {
  return p->n_kv_heads == s->Hkv && p->head_dim == s->d && p->dtype == s->dtype;
}

void lru_unlink(hga_kv_store* s, int32_t i) {
  const int32_t a = s->prev[i], b = s->next[i];
  if (a >= 0) s->next[a] = b; else if (s->lru_head == i) s->lru_head = b;
  if (b >= 0) s->prev[b] = a; else if (s->lru_tail == i) s->lru_tail = a;
  s->prev[i] = s->next[i] = -1;
}

void lru_push_front(hga_kv_store* s, int32_t i) {
  s->prev[i] = -1;
  s->next[i] = s->lru_head;
  if (s->lru_head >= 0) s->prev[s->lru_head] = i;
  s->lru_head = i;
  if (s->lru_tail < 0) s->lru_tail = i;
}

}  // namespace

extern "C" {

hga_status hga_store_open(const char* path, const hga_params* p, int64_t t_cap,
                          int64_t page_tokens, int32_t flags, hga_kv_store** out) {
  if (out) *out = nullptr;
  if (!path || !p || !out) return HGA_ERR_INVALID_ARG;
  hga_status st = hga_validate_params(p);
  if (st != HGA_OK) return st;
  if (t_cap <= 0 || page_tokens <= 0 || page_tokens % p->group || (flags & ~3))
    return HGA_ERR_INVALID_ARG;
  const int64_t elem = p->dtype == HGA_BF16 ? 2 : 4;
  const int64_t half = page_tokens * p->head_dim * elem;
  const bool direct = (flags & HGA_STORE_DIRECT) != 0;
  if (direct && (2 * half) % 4096) return HGA_ERR_INVALID_ARG;
  const int64_t n_pages = (t_cap + page_tokens - 1) / page_tokens;
  const int64_t size = (int64_t)p->n_kv_heads * n_pages * 2 * half;

  const bool create = (flags & HGA_STORE_CREATE) != 0;
  int fd = ::open(path, O_RDWR | O_CLOEXEC | (create ? O_CREAT | O_TRUNC : 0), 0644);
  if (fd < 0) return HGA_ERR_IO;
  if (create) {
    if (::ftruncate(fd, (off_t)size) != 0) {
      ::close(fd);
      return HGA_ERR_IO;
    }
  } else {
    struct stat sb;
    if (::fstat(fd, &sb) != 0 || (int64_t)sb.st_size < size) {
      ::close(fd);
      return HGA_ERR_IO;
    }
  }
  int fd_r = fd;
  if (direct) {
    fd_r = ::open(path, O_RDONLY | O_CLOEXEC | O_DIRECT);
    if (fd_r < 0) {
      ::close(fd);
      return HGA_ERR_IO;
    }
  }
  hga_kv_store* s = new (std::nothrow) hga_kv_store();
  if (!s) {
    if (fd_r != fd) ::close(fd_r);
    ::close(fd);
    return HGA_ERR_INVALID_ARG;
  }
  s->path = path;
  s->fd_write = fd;
  s->fd_read = fd_r;
  s->direct = direct;
  s->dtype = p->dtype;
  s->Hkv = p->n_kv_heads;
  s->d = p->head_dim;
  s->elem = elem;
  s->t_cap = t_cap;
  s->page_tokens = page_tokens;
  s->n_pages = n_pages;
  s->half_bytes = half;
  s->page_bytes = 2 * half;
  *out = s;
  return HGA_OK;
}

hga_status hga_store_close(hga_kv_store* s) {
  if (!s) return HGA_OK;
  bool ok = true;
  if (s->fd_read >= 0 && s->fd_read != s->fd_write) ok &= ::close(s->fd_read) == 0;
  if (s->fd_write >= 0) ok &= ::close(s->fd_write) == 0;
  delete s;
  return ok ? HGA_OK : HGA_ERR_IO;
}

hga_status hga_store_attach_cache(hga_kv_store* s, void* cache, int64_t cache_pages,
                                  int32_t* page_table) {
  if (!s || !cache || !page_table || cache_pages <= 0 || cache_pages > 0x7fffffff)
    return HGA_ERR_INVALID_ARG;
  // 16-byte rows for the gather kernel's vector copies; 4096 for O_DIRECT reads
  if (reinterpret_cast<uintptr_t>(cache) % (s->direct ? 4096 : 16)) return HGA_ERR_INVALID_ARG;
  const int64_t n_global = s->Hkv * s->n_pages;
  try {                                         // no C++ exception crosses the C ABI
    s->slot_page.assign((size_t)cache_pages, -1);
    s->prev.assign((size_t)cache_pages, -1);
    s->next.assign((size_t)cache_pages, -1);
    s->slot_step.assign((size_t)cache_pages, 0);
    s->page_step.assign((size_t)n_global, 0);
    s->free_slots.resize((size_t)cache_pages);
  } catch (...) {
    s->cache = nullptr;
    s->page_table = nullptr;
    s->cache_pages = 0;
    return HGA_ERR_INVALID_ARG;
  }
  s->cache = static_cast<char*>(cache);
  s->cache_pages = cache_pages;
  s->page_table = page_table;
  for (int64_t i = 0; i < cache_pages; ++i) s->free_slots[(size_t)i] = (int32_t)(cache_pages - 1 - i);
  s->lru_head = s->lru_tail = -1;
  s->step = 0;
  std::fill(page_table, page_table + n_global, -1);
  return HGA_OK;
}

hga_status hga_store_append(hga_kv_store* s, const void* k, const void* v, int64_t n) {
  if (!s || n < 0 || s->length + n > s->t_cap) return HGA_ERR_INVALID_ARG;
  if (n == 0) return HGA_OK;
  if (!k || !v) return HGA_ERR_INVALID_ARG;
  const int64_t row = s->d * s->elem;
  const int64_t t0 = s->length, t1 = s->length + n;
  for (int64_t h = 0; h < s->Hkv; ++h) {
    for (int64_t t = t0; t < t1;) {
      const int64_t pg = t / s->page_tokens, t_in = t % s->page_tokens;
      const int64_t cnt = std::min(s->page_tokens - t_in, t1 - t);
      const int64_t src = (h * n + (t - t0)) * row;
      const int64_t page_off = (h * s->n_pages + pg) * s->page_bytes;
      const int64_t in_off = t_in * row;
      const char* ks = static_cast<const char*>(k) + src;
      const char* vs = static_cast<const char*>(v) + src;
      if (!pwrite_full(s->fd_write, ks, cnt * row, page_off + in_off) ||
          !pwrite_full(s->fd_write, vs, cnt * row, page_off + s->half_bytes + in_off))
        return HGA_ERR_IO;
      if (s->page_table) {                      // write through to a cached copy
        const int32_t slot = s->page_table[h * s->n_pages + pg];
        if (slot >= 0) {
          char* base = s->cache + (int64_t)slot * s->page_bytes;
          memcpy(base + in_off, ks, (size_t)(cnt * row));
          memcpy(base + s->half_bytes + in_off, vs, (size_t)(cnt * row));
        }
      }
      t += cnt;
    }
  }
  s->length = t1;
  return HGA_OK;
}

hga_status hga_store_set_length(hga_kv_store* s, int64_t length) {
  if (!s || length < 0 || length > s->t_cap) return HGA_ERR_INVALID_ARG;
  s->length = length;
  return HGA_OK;
}

int64_t hga_store_length(const hga_kv_store* s) { return s ? s->length : -1; }
int64_t hga_store_page_bytes(const hga_kv_store* s) { return s ? s->page_bytes : -1; }
int64_t hga_store_pages_per_head(const hga_kv_store* s) { return s ? s->n_pages : -1; }

hga_status hga_store_read(hga_kv_store* s, int64_t t_begin, int64_t t_end, void* k, void* v) {
  if (!s || t_begin < 0 || t_begin > t_end || t_end > s->t_cap) return HGA_ERR_INVALID_ARG;
  const int64_t n = t_end - t_begin;
  if (n == 0) return HGA_OK;
  if (!k || !v) return HGA_ERR_INVALID_ARG;
  const int64_t row = s->d * s->elem;
  for (int64_t h = 0; h < s->Hkv; ++h) {
    for (int64_t t = t_begin; t < t_end;) {
      const int64_t pg = t / s->page_tokens, t_in = t % s->page_tokens;
      const int64_t cnt = std::min(s->page_tokens - t_in, t_end - t);
      const int64_t dst = (h * n + (t - t_begin)) * row;
      const int64_t off = (h * s->n_pages + pg) * s->page_bytes + t_in * row;
      if (!pread_full(s->fd_write, static_cast<char*>(k) + dst, cnt * row, off) ||
          !pread_full(s->fd_write, static_cast<char*>(v) + dst, cnt * row, off + s->half_bytes))
        return HGA_ERR_IO;
      t += cnt;
    }
  }
  return HGA_OK;
}

hga_status hga_store_prepare(hga_kv_store* s, const hga_params* p, int64_t q_start,
                             int64_t n_q, int64_t t_hist, const int32_t* group_idx,
                             const int32_t* group_cnt, int32_t io_threads,
                             hga_store_stats* stats) {
  if (stats) *stats = hga_store_stats{};
  if (!s || !p || !s->page_table || io_threads < 1) return HGA_ERR_INVALID_ARG;
  hga_status st = hga_validate_params(p);
  if (st != HGA_OK) return st;
  if (!same_layout(s, p)) return HGA_ERR_INVALID_ARG;
  if (q_start < 0 || n_q < 0 || q_start + n_q > s->t_cap) return HGA_ERR_INVALID_ARG;
  if (t_hist < 0 || t_hist > q_start || t_hist % p->group || t_hist > s->length)
    return HGA_ERR_INVALID_ARG;
  if (n_q == 0) return HGA_OK;
  if (!group_idx || !group_cnt) return HGA_ERR_INVALID_ARG;
  const int64_t cap_g = hga_index_capacity(p, s->t_cap, 1);
  if (cap_g < 0) return HGA_ERR_INVALID_ARG;
  const int64_t n_blocks = (n_q + p->qblock - 1) / p->qblock;
  const int64_t g = p->group;

  if (++s->step == 0) {                         // stamp wrap-around: restart the stamps
    std::fill(s->slot_step.begin(), s->slot_step.end(), 0u);
    std::fill(s->page_step.begin(), s->page_step.end(), 0u);
    s->step = 1;
  }
  const uint32_t step = s->step;
  hga_store_stats c{};
  std::vector<int64_t> missing;
  std::vector<int32_t> slots;
  std::vector<char> ok;
  std::vector<std::pair<size_t, size_t>> runs;   // (first index in missing, pages)
  try {                                         // reserve up front: no throw below
    missing.reserve((size_t)std::min<int64_t>(s->cache_pages, s->Hkv * s->n_pages));
  } catch (...) {
    return HGA_ERR_INVALID_ARG;
  }
  for (int64_t h = 0; h < s->Hkv; ++h) {
    for (int64_t b = 0; b < n_blocks; ++b) {
      const int64_t b0 = q_start + b * p->qblock;
      const int64_t sink_end = std::min<int64_t>(p->sink, b0);
      const int64_t n_s = sink_end / g;
      int64_t n_r = group_cnt[h * n_blocks + b];
      if (n_r < 0 || n_r > cap_g) n_r = 0;      // the gather kernel skips these too
      const int32_t* routed = group_idx + (h * n_blocks + b) * cap_g;
      const int64_t loc_lo = std::max<int64_t>(sink_end, b0 - p->local);
      const int64_t n_l = (b0 - loc_lo) / g;
      for (int64_t i = 0; i < n_s + n_r + n_l; ++i) {
        int64_t j;
        if (i < n_s) j = i;
        else if (i < n_s + n_r) j = routed[i - n_s];
        else j = loc_lo / g + (i - n_s - n_r);
        if (j < 0 || (j + 1) * g > t_hist) continue;
        const int64_t gp = h * s->n_pages + (j * g) / s->page_tokens;
        if (s->page_step[(size_t)gp] == step) continue;
        s->page_step[(size_t)gp] = step;
        ++c.pages_needed;
        const int32_t slot = s->page_table[gp];
        if (slot >= 0) {
          ++c.hits;
          s->slot_step[(size_t)slot] = step;
          lru_unlink(s, slot);
          lru_push_front(s, slot);
        } else if (missing.size() < missing.capacity()) {
          missing.push_back(gp);
        }   // else: more misses than slots, so pages_needed > cache_pages below
      }
    }
  }
  if (c.pages_needed > s->cache_pages) {
    if (stats) *stats = c;
    return HGA_ERR_CAPACITY;
  }
  std::sort(missing.begin(), missing.end());    // file order, for runs of adjacent pages

  // slots for the missing pages: free ones first, then the least recently
  // used pages this step does not need (they sit at the tail of the list)
  try {
    slots.resize(missing.size());
    ok.assign(missing.size(), 0);
  } catch (...) {
    if (stats) *stats = c;
    return HGA_ERR_INVALID_ARG;
  }
  for (size_t i = 0; i < missing.size(); ++i) {
    int32_t slot;
    if (!s->free_slots.empty()) {
      slot = s->free_slots.back();
      s->free_slots.pop_back();
    } else {
      slot = s->lru_tail;
      if (slot < 0 || s->slot_step[(size_t)slot] == step) {   // cannot happen after the count check
        if (stats) *stats = c;
        for (size_t r = 0; r < i; ++r) {
          s->slot_page[(size_t)slots[r]] = -1;
          lru_unlink(s, slots[r]);
          s->free_slots.push_back(slots[r]);
        }
        return HGA_ERR_CAPACITY;
      }
      s->page_table[s->slot_page[(size_t)slot]] = -1;
      lru_unlink(s, slot);
      ++c.evictions;
    }
    s->slot_page[(size_t)slot] = missing[i];
    s->slot_step[(size_t)slot] = step;
    lru_push_front(s, slot);
    slots[i] = slot;
  }

  // reads, several in flight: runs of pages adjacent in the file (missing is
  // sorted) go into one vectored read of up to 1 MiB, each page to its slot
  const size_t max_run = (size_t)std::max<int64_t>(
      1, std::min<int64_t>(kMaxRunPages, (1 << 20) / s->page_bytes));
  try {
    for (size_t i = 0; i < missing.size();) {
      size_t n = 1;
      while (i + n < missing.size() && n < max_run && missing[i + n] == missing[i] + (int64_t)n) ++n;
      runs.emplace_back(i, n);
      i += n;
    }
  } catch (...) {
    runs.clear();
    for (size_t i = 0; i < missing.size(); ++i) {
      s->slot_page[(size_t)slots[i]] = -1;
      lru_unlink(s, slots[i]);
      s->free_slots.push_back(slots[i]);
    }
    if (stats) *stats = c;
    return HGA_ERR_INVALID_ARG;
  }
  auto worker = [&](std::atomic<size_t>* next) {
    struct iovec iov[kMaxRunPages];
    for (size_t r; (r = next->fetch_add(1)) < runs.size();) {
      const size_t i0 = runs[r].first, n = runs[r].second;
      for (size_t j = 0; j < n; ++j) {
        iov[j].iov_base = s->cache + (int64_t)slots[i0 + j] * s->page_bytes;
        iov[j].iov_len = (size_t)s->page_bytes;
      }
      const char good = preadv_full(s->fd_read, iov, (int)n, missing[i0] * s->page_bytes);
      for (size_t j = 0; j < n; ++j) ok[i0 + j] = good;
    }
  };
  std::atomic<size_t> next{0};
  const size_t n_thr = std::min<size_t>((size_t)io_threads, runs.size());
  if (n_thr <= 1) {
    worker(&next);
  } else {
    std::vector<std::thread> pool;
    try {                                       // fewer threads if the system refuses some
      pool.reserve(n_thr - 1);
      for (size_t t = 1; t < n_thr; ++t) pool.emplace_back(worker, &next);
    } catch (...) {
    }
    worker(&next);
    for (auto& th : pool) th.join();
  }
  for (size_t i = 0; i < missing.size(); ++i) {
    if (ok[i]) {
      s->page_table[missing[i]] = slots[i];
      ++c.misses;
      c.bytes_read += s->page_bytes;
    } else {
      s->slot_page[(size_t)slots[i]] = -1;
      lru_unlink(s, slots[i]);
      s->free_slots.push_back(slots[i]);
      st = HGA_ERR_IO;
    }
  }
  if (stats) *stats = c;
  return st;
}

}  // extern "C"
