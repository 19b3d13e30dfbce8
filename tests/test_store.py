"""File-backed K/V store, host side (no GPU): the file layout, appends and
reads, and the page cache that hga_store_prepare fills for a step.

"Long-Context Fine-Tuning with Limited VRAM", section 2.2: besides RAM-backed
history there is a filesystem store in which RAM is a bounded page cache over
disk.  The pages a step needs are fixed by the routing (section 2.1: sink and
local windows plus the routed groups); the expected sets below are built from
that definition, independently of the library's enumeration."""
import ctypes

import numpy as np
import pytest
import torch

import hga_inputs as gi

PT = 64          # page tokens in most tests


@pytest.fixture(scope="module")
def hga():
    from long_context_hga_b200 import build
    build.build()
    from long_context_hga_b200 import hga as mod
    return mod


def _params(hga, **kw):
    w = gi.TIERED_128K.with_(**kw)
    return hga.Params.from_workload(w), w


def _kv(w, n, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(w.n_kv_heads, n, w.head_dim, generator=g).to(torch.bfloat16)
    v = torch.randn(w.n_kv_heads, n, w.head_dim, generator=g).to(torch.bfloat16)
    return k, v


def _bits(t):
    return t.contiguous().view(torch.int16)


def _store(hga, p, path, t_cap, cache_pages, page_tokens=PT, direct=False):
    return hga.KVStore(p, str(path), t_cap, page_tokens, cache_pages, create=True,
                       direct=direct, pin=False)


def _needed_pages(p, w, q_start, n_q, t_hist, gidx, gcnt, page_tokens):
    """(KV head, page) pairs whose tokens a step reads from history: per
    (block, KV head) the sink groups, the routed groups and the local-window
    groups, below t_hist."""
    g = w.group
    need = set()
    n_blocks = -(-n_q // w.qblock)
    for h in range(w.n_kv_heads):
        for b in range(n_blocks):
            b0 = q_start + b * w.qblock
            sink_end = min(w.sink, b0)
            groups = list(range(sink_end // g))
            groups += [int(x) for x in gidx[h, b, :gcnt[h, b]]]
            groups += list(range(max(sink_end, b0 - w.local) // g, b0 // g))
            for j in groups:
                if 0 <= j and (j + 1) * g <= t_hist:
                    need.add((h, j * g // page_tokens))
    return need


def _routing(w, p, hga, q_start, n_q, t_hist, seed, t_cap):
    """Random routed groups inside the history (distinct per block)."""
    rng = np.random.default_rng(seed)
    n_blocks = -(-n_q // w.qblock)
    cap_g = hga.index_capacity(p, t_cap, 1)
    gidx = np.full((w.n_kv_heads, n_blocks, max(cap_g, 1)), -1, dtype=np.int32)
    gcnt = np.zeros((w.n_kv_heads, n_blocks), dtype=np.int32)
    for h in range(w.n_kv_heads):
        for b in range(n_blocks):
            n = int(rng.integers(0, cap_g + 1))
            gidx[h, b, :n] = np.sort(rng.choice(t_hist // w.group, n, replace=False))
            gcnt[h, b] = n
    return gidx, gcnt


def _prepare(store, p, q_start, n_q, t_hist, gidx, gcnt, io_threads=4):
    return store.prepare(p, q_start, n_q, t_hist, torch.from_numpy(gidx),
                         torch.from_numpy(gcnt), io_threads)


def _check_cache(store, w, k_all, v_all, pages):
    """Every listed page is resident and its slot holds the page's K then V."""
    cache = store.cache.view(torch.int16).view(store.cache_pages, 2, store.page_tokens,
                                               w.head_dim)
    pt = store.page_tokens
    for h, n in pages:
        slot = int(store.page_table[h, n])
        assert 0 <= slot < store.cache_pages, (h, n, slot)
        t0, t1 = n * pt, min((n + 1) * pt, k_all.shape[1])
        assert torch.equal(cache[slot, 0, :t1 - t0], _bits(k_all[h, t0:t1]))
        assert torch.equal(cache[slot, 1, :t1 - t0], _bits(v_all[h, t0:t1]))


def test_append_read_roundtrip_and_file_layout(hga, tmp_path):
    p, w = _params(hga)
    t_cap = 1000                                     # ragged last page
    path = tmp_path / "kv.bin"
    s = _store(hga, p, path, t_cap, cache_pages=4)
    assert s.n_pages == -(-t_cap // PT)
    assert s.page_bytes == 2 * PT * w.head_dim * 2
    k, v = _kv(w, 937, 1)
    off = 0
    for n in (100, 37, 0, 300, 500):                 # pieces that straddle pages
        s.append(k[:, off:off + n], v[:, off:off + n])
        off += n
    assert s.length == 937
    rk, rv = s.read(0, 937)
    assert torch.equal(_bits(rk), _bits(k)) and torch.equal(_bits(rv), _bits(v))
    rk, rv = s.read(123, 611)
    assert torch.equal(_bits(rk), _bits(k[:, 123:611]))
    assert torch.equal(_bits(rv), _bits(v[:, 123:611]))
    tk, tv = s.read(937, 1000)                       # never appended: zeros
    assert not _bits(tk).any() and not _bits(tv).any()
    s.close()
    # the documented layout: page (h, n) at (h * n_pages + n) * page_bytes, K then V
    raw = np.fromfile(path, dtype=np.int16).reshape(w.n_kv_heads, -(-t_cap // PT), 2, PT,
                                                   w.head_dim)
    kb, vb = _bits(k).numpy(), _bits(v).numpy()
    for h in (0, 5, 7):
        for n in (0, 3, 14):
            t0, t1 = n * PT, min((n + 1) * PT, 937)
            assert np.array_equal(raw[h, n, 0, :t1 - t0], kb[h, t0:t1])
            assert np.array_equal(raw[h, n, 1, :t1 - t0], vb[h, t0:t1])


def test_reopen_existing_file(hga, tmp_path):
    p, w = _params(hga)
    path = tmp_path / "kv.bin"
    s = _store(hga, p, path, 512, cache_pages=2)
    k, v = _kv(w, 512, 2)
    s.append(k, v)
    s.close()
    s2 = hga.KVStore(p, str(path), 512, PT, 2, create=False, pin=False)
    assert s2.length == 0
    s2.set_length(512)
    rk, rv = s2.read(0, 512)
    assert torch.equal(_bits(rk), _bits(k)) and torch.equal(_bits(rv), _bits(v))
    with pytest.raises(hga.HgaError):
        hga.KVStore(p, str(path), 1024, PT, 2, create=False, pin=False)   # file too short
    with pytest.raises(hga.HgaError):
        hga.KVStore(p, str(tmp_path / "missing.bin"), 512, PT, 2, create=False, pin=False)


@pytest.mark.parametrize("page_tokens", [64, 8, 256])
def test_prepare_loads_exactly_the_needed_pages(hga, tmp_path, page_tokens):
    p, w = _params(hga, top_chunks=8, top_groups=16, sink=64, local=128)
    t_cap, q_start, n_q = 4096, 3072, 256
    t_hist = q_start
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=4096,
               page_tokens=page_tokens)
    k, v = _kv(w, t_hist, 3)
    s.append(k, v)
    gidx, gcnt = _routing(w, p, hga, q_start, n_q, t_hist, 4, t_cap)
    need = _needed_pages(p, w, q_start, n_q, t_hist, gidx, gcnt, page_tokens)
    st = _prepare(s, p, q_start, n_q, t_hist, gidx, gcnt)
    assert st["pages_needed"] == len(need) == st["misses"]
    assert st["hits"] == 0 and st["evictions"] == 0
    assert st["bytes_read"] == len(need) * s.page_bytes
    resident = {(h, n) for h in range(w.n_kv_heads) for n in range(s.n_pages)
                if s.page_table[h, n] >= 0}
    assert resident == need
    _check_cache(s, w, k, v, need)
    slots = [int(s.page_table[h, n]) for h, n in need]
    assert len(set(slots)) == len(slots)
    st2 = _prepare(s, p, q_start, n_q, t_hist, gidx, gcnt)     # same step again: all hits
    assert st2["hits"] == len(need) and st2["misses"] == 0 and st2["bytes_read"] == 0


def test_lru_eviction_order(hga, tmp_path):
    """Cache of 3 pages; steps that each need one routed page: A, B, C, A, D.
    D must evict B (least recently used), not A."""
    p, w = _params(hga, n_kv_heads=1, n_q_heads=4, top_chunks=1, top_groups=1, sink=0,
                   local=0)
    t_cap, q_start, n_q = 1024, 960, 64
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=3)
    k, v = _kv(w, q_start, 5)
    s.append(k, v)
    cap_g = hga.index_capacity(p, t_cap, 1)
    assert cap_g == 1

    def step(page):
        gidx = np.array([[[page * PT // w.group + 3]]], dtype=np.int32)
        gcnt = np.array([[1]], dtype=np.int32)
        return _prepare(s, p, q_start, n_q, q_start, gidx, gcnt)

    for page, hit in ((0, 0), (1, 0), (2, 0), (0, 1)):
        st = step(page)
        assert st["pages_needed"] == 1 and st["hits"] == hit and st["evictions"] == 0
    st = step(3)
    assert st["misses"] == 1 and st["evictions"] == 1
    assert s.page_table[0, 1] == -1                       # B evicted
    for n in (0, 2, 3):
        assert s.page_table[0, n] >= 0
    _check_cache(s, w, k, v, {(0, 0), (0, 2), (0, 3)})
    st = step(1)                                          # B again: evicts C (LRU now)
    assert st["misses"] == 1 and st["evictions"] == 1 and s.page_table[0, 2] == -1


def test_eviction_never_drops_a_page_the_step_needs(hga, tmp_path):
    p, w = _params(hga, top_chunks=8, top_groups=16, sink=64, local=128)
    t_cap, q_start, n_q = 4096, 3072, 256
    s0 = _store(hga, p, tmp_path / "probe.bin", t_cap, cache_pages=4096)
    k, v = _kv(w, q_start, 6)
    s0.append(k, v)
    steps = [_routing(w, p, hga, q_start, n_q, q_start, 10 + i, t_cap) for i in range(4)]
    needs = [_needed_pages(p, w, q_start, n_q, q_start, a, b, PT) for a, b in steps]
    cap = max(len(n) for n in needs)                      # exactly one step's worth
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=cap)
    s.append(k, v)
    prev = set()
    for (gidx, gcnt), need in zip(steps, needs):
        st = _prepare(s, p, q_start, n_q, q_start, gidx, gcnt)
        assert st["pages_needed"] == len(need)
        assert st["hits"] == len(need & prev)
        assert st["misses"] == len(need - prev)
        _check_cache(s, w, k, v, need)
        prev = {(h, n) for h in range(w.n_kv_heads) for n in range(s.n_pages)
                if s.page_table[h, n] >= 0}
        assert need <= prev and len(prev) <= cap


def test_capacity_error(hga, tmp_path):
    p, w = _params(hga, top_chunks=8, top_groups=16, sink=64, local=128)
    t_cap, q_start, n_q = 4096, 3072, 256
    k, v = _kv(w, q_start, 7)
    gidx, gcnt = _routing(w, p, hga, q_start, n_q, q_start, 8, t_cap)
    need = _needed_pages(p, w, q_start, n_q, q_start, gidx, gcnt, PT)
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=len(need) - 1)
    s.append(k, v)
    with pytest.raises(hga.HgaError) as e:
        _prepare(s, p, q_start, n_q, q_start, gidx, gcnt)
    assert e.value.code == hga.HGA_ERR_CAPACITY
    assert not (s.page_table >= 0).any()                  # nothing half-loaded


def test_append_writes_through_to_cached_pages(hga, tmp_path):
    p, w = _params(hga, n_kv_heads=2, n_q_heads=8, top_chunks=1, top_groups=1, sink=0,
                   local=0)
    t_cap = 1024
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=4)
    k, v = _kv(w, 200, 9)
    s.append(k[:, :160], v[:, :160])                      # page 2 half written
    gidx = np.array([[[16]], [[17]]], dtype=np.int32)      # groups in page 2 (tokens 128..)
    gcnt = np.ones((2, 1), dtype=np.int32)
    _prepare(s, p, 192, 64, 152, gidx, gcnt)
    assert (s.page_table[:, 2] >= 0).all()
    s.append(k[:, 160:], v[:, 160:])                      # the rest of page 2, and page 3
    _check_cache(s, w, k, v, {(0, 2), (1, 2)})


def test_parallel_reads_match_serial(hga, tmp_path):
    p, w = _params(hga, top_chunks=16, top_groups=32, sink=64, local=256)
    t_cap, q_start, n_q = 8192, 6144, 512
    k, v = _kv(w, q_start, 11)
    gidx, gcnt = _routing(w, p, hga, q_start, n_q, q_start, 12, t_cap)
    need = _needed_pages(p, w, q_start, n_q, q_start, gidx, gcnt, PT)
    for threads in (1, 8):
        s = _store(hga, p, tmp_path / f"kv{threads}.bin", t_cap, cache_pages=len(need))
        s.append(k, v)
        st = _prepare(s, p, q_start, n_q, q_start, gidx, gcnt, io_threads=threads)
        assert st["misses"] == len(need)
        _check_cache(s, w, k, v, need)


def test_direct_io_when_the_filesystem_allows_it(hga, tmp_path):
    p, w = _params(hga, top_chunks=8, top_groups=16, sink=64, local=128)
    t_cap, q_start, n_q = 4096, 3072, 256
    try:
        s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=2048, direct=True)
    except hga.HgaError as e:
        assert e.code == hga.HGA_ERR_IO
        pytest.skip("O_DIRECT refused by this filesystem")
    k, v = _kv(w, q_start, 13)
    s.append(k, v)                                        # buffered writes, direct reads
    gidx, gcnt = _routing(w, p, hga, q_start, n_q, q_start, 14, t_cap)
    need = _needed_pages(p, w, q_start, n_q, q_start, gidx, gcnt, PT)
    st = _prepare(s, p, q_start, n_q, q_start, gidx, gcnt)
    assert st["misses"] == len(need)
    _check_cache(s, w, k, v, need)


def test_argument_checks(hga, tmp_path):
    p, w = _params(hga)
    L = hga.LIB
    h = ctypes.c_void_p()
    path = str(tmp_path / "kv.bin").encode()
    E = hga.HGA_ERR_INVALID_ARG
    assert L.hga_store_open(path, ctypes.byref(p.c()), 1024, 12, 1, ctypes.byref(h)) == E
    assert L.hga_store_open(path, ctypes.byref(p.c()), 0, 64, 1, ctypes.byref(h)) == E
    assert L.hga_store_open(path, ctypes.byref(p.c()), 1024, 64, 4, ctypes.byref(h)) == E
    assert L.hga_store_open(None, ctypes.byref(p.c()), 1024, 64, 1, ctypes.byref(h)) == E
    assert h.value is None
    # direct reads need 4096-byte pages: 8 tokens x 128 x 2 B x 2 = 4096 passes, fp32 d=64
    # with 8 tokens = 4096 too; bf16 d=64 with 8 tokens = 2048 does not
    p64, _ = _params(hga, head_dim=64)
    assert L.hga_store_open(path, ctypes.byref(p64.c()), 1024, 8, 3, ctypes.byref(h)) == E
    s = _store(hga, p, tmp_path / "kv.bin", 1024, cache_pages=2)
    k, v = _kv(w, 64, 15)
    assert L.hga_store_append(s.handle, hga._ptr(k), hga._ptr(v), 2000) == E   # past t_cap
    assert L.hga_store_append(s.handle, None, None, 64) == E
    assert L.hga_store_set_length(s.handle, 1025) == E
    assert L.hga_store_read(s.handle, 10, 5, None, None) == E
    assert L.hga_store_attach_cache(s.handle, None, 2, hga._ptr(s.page_table)) == E
    misaligned = s.cache[8:8 + s.page_bytes]
    assert L.hga_store_attach_cache(s.handle, hga._ptr(misaligned), 1,
                                    hga._ptr(s.page_table)) == E
    s.append(k, v)
    gidx = np.zeros((w.n_kv_heads, 1, 64), dtype=np.int32)
    gcnt = np.zeros((w.n_kv_heads, 1), dtype=np.int32)
    with pytest.raises(hga.HgaError):                     # t_hist beyond the length
        _prepare(s, p, 128, 64, 128, gidx, gcnt)
    with pytest.raises(hga.HgaError):                     # t_hist > q_start
        _prepare(s, p, 56, 64, 64, gidx, gcnt)
    with pytest.raises(hga.HgaError):                     # io_threads < 1
        _prepare(s, p, 64, 64, 64, gidx, gcnt, io_threads=0)
    p_other, _ = _params(hga, n_kv_heads=4, n_q_heads=16)
    with pytest.raises(hga.HgaError):                     # another layout
        _prepare(s, p_other, 64, 64, 64, gidx[:4], gcnt[:4])
    assert L.hga_store_length(None) == -1
    assert L.hga_store_close(None) == hga.HGA_OK
    assert _prepare(s, p, 64, 0, 64, gidx, gcnt)["pages_needed"] == 0


def test_replacement_policy_over_many_random_steps(hga, tmp_path):
    """Random steps over one history with a cache of about a third of it.
    After every step: the step's pages are resident and hold their bytes,
    residency never exceeds the cache, nothing leaves without a reason (a
    resident page disappears only when the step had misses to place), and
    eviction follows least-recent use by step: every evicted page was last
    used no later than every retained page the step did not need."""
    p, w = _params(hga, n_kv_heads=2, n_q_heads=4, top_chunks=4, top_groups=6, sink=64,
                   local=64)
    t_cap = 2048
    q_starts = [1024, 1536, 1984]
    k, v = _kv(w, 1024, 21)
    pt = 8                                              # one group per page
    hist_pages = w.n_kv_heads * 1024 // pt
    s = _store(hga, p, tmp_path / "kv.bin", t_cap, cache_pages=hist_pages // 3,
               page_tokens=pt)
    s.append(k, v)
    rng = np.random.default_rng(22)
    last_use = {}
    resident = set()
    done = evictions = 0
    for step in range(1, 41):
        q_start = int(rng.choice(q_starts))
        n_q = int(rng.integers(1, 3)) * 64 if q_start < 1984 else 64
        n_q = min(n_q, t_cap - q_start)
        gidx, gcnt = _routing(w, p, hga, q_start, n_q, 1024, 100 + step, t_cap)
        need = _needed_pages(p, w, q_start, n_q, 1024, gidx, gcnt, pt)
        if len(need) > s.cache_pages:
            with pytest.raises(hga.HgaError) as e:
                _prepare(s, p, q_start, n_q, 1024, gidx, gcnt)
            assert e.value.code == hga.HGA_ERR_CAPACITY
            continue
        st = _prepare(s, p, q_start, n_q, 1024, gidx, gcnt, io_threads=3)
        now = {(h, n) for h in range(w.n_kv_heads) for n in range(s.n_pages)
               if s.page_table[h, n] >= 0}
        assert need <= now and len(now) <= s.cache_pages
        assert st["hits"] == len(need & resident)
        assert st["misses"] == len(need - resident)
        evicted = resident - now
        assert now - need <= resident                     # no stray page appears
        assert st["evictions"] == len(evicted)
        if evicted:
            assert st["misses"] > 0
            kept_old = now - need
            if kept_old:
                assert max(last_use[x] for x in evicted) <= min(last_use[x] for x in kept_old)
        for x in need:
            last_use[x] = step
        resident = now
        done += 1
        evictions += st["evictions"]
        if step % 8 == 0:
            _check_cache(s, w, k, v, need)
    assert done >= 30 and evictions > 0, (done, evictions)
    slots = s.page_table[s.page_table >= 0]
    assert len(set(slots.tolist())) == len(slots)         # one page per slot


def test_fp32_store_with_head_dim_64(hga, tmp_path):
    """The layout and the cache for 4-byte elements and d = 64."""
    w = gi.TINY_FP32.with_(T=2048, q0=1536)
    p = hga.Params.from_workload(w)
    g = torch.Generator().manual_seed(31)
    k = torch.randn(w.n_kv_heads, 1536, w.head_dim, generator=g)
    v = torch.randn(w.n_kv_heads, 1536, w.head_dim, generator=g)
    s = _store(hga, p, tmp_path / "kv.bin", w.T, cache_pages=64)
    assert s.page_bytes == 2 * PT * w.head_dim * 4
    s.append(k[:, :700], v[:, :700])
    s.append(k[:, 700:], v[:, 700:])
    rk, rv = s.read(5, 1530)
    assert torch.equal(rk, k[:, 5:1530]) and torch.equal(rv, v[:, 5:1530])
    gidx, gcnt = _routing(w, p, hga, w.q0, w.Tq, w.q0, 32, w.T)
    need = _needed_pages(p, w, w.q0, w.Tq, w.q0, gidx, gcnt, PT)
    st = _prepare(s, p, w.q0, w.Tq, w.q0, gidx, gcnt)
    assert st["misses"] == len(need) > 0
    cache = s.cache.view(torch.float32).view(s.cache_pages, 2, PT, w.head_dim)
    for h, n in need:
        slot = int(s.page_table[h, n])
        assert torch.equal(cache[slot, 0], k[h, n * PT:(n + 1) * PT])
        assert torch.equal(cache[slot, 1], v[h, n * PT:(n + 1) * PT])
