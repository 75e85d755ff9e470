"""The state cache's page allocator (csa_page_alloc_*, csa_state_pages_needed) on the CPU.

- FIFO hand-out and all-or-nothing reservations on a worked example;
- argument checks;
- csa_state_pages_needed against its closed form at block boundaries (CSA m = 4 with
  32-entry pages, HCA m' = 128 with one-entry pages);
- driven the way a decode loop drives it (reserve the pages of the entries a token may
  finish before appending it; give a finished request's pages back), the page tables equal
  those of the oracle's state cache (oracle/state_cache.py), which takes a page from its
  shared pool when an entry opens a new block and gives a request's pages back in order;
  both run out of pages at the same token.
"""
import ctypes

import numpy as np
import pytest

import long_context_sparse_08_b200 as csa
from oracle import state_cache as SC


def test_fifo_handout_and_all_or_nothing():
    a = csa.PageAlloc(10, 3, 4)
    assert a.free_pages == 10 and (a.table == -1).all()
    a.reserve(0, 2)
    a.reserve(1, 3)
    a.reserve(0, 2)  # already mapped: nothing taken
    a.reserve(0, 1)  # fewer than mapped: nothing changes
    assert a.table.tolist() == [[0, 1, -1, -1], [2, 3, 4, -1], [-1, -1, -1, -1]]
    a.reserve(2, 4)
    assert a.free_pages == 1
    with pytest.raises(csa.CsaError) as e:
        a.reserve(0, 4)  # two more needed, one free
    assert e.value.status == csa.CSA_ERR_NO_PAGES
    assert a.table[0].tolist() == [0, 1, -1, -1] and a.free_pages == 1 and a.mapped(0) == 2
    a.release(1)  # pages 2, 3, 4 join the back of the free list after 9
    assert a.table[1].tolist() == [-1] * 4 and a.mapped(1) == 0 and a.free_pages == 4
    a.reserve(0, 4)
    assert a.table[0].tolist() == [0, 1, 9, 2]
    a.reserve(1, 2)
    assert a.table[1].tolist() == [3, 4, -1, -1] and a.free_pages == 0
    a.release(2)
    a.release(2)  # releasing an empty row is a no-op
    assert a.free_pages == 4
    a.close()


def test_argument_checks():
    L = csa.lib()
    h = ctypes.c_void_p()
    assert L.csa_page_alloc_create(0, 2, 4, ctypes.byref(h)) == csa.CSA_ERR_INVALID_ARG
    assert not h.value
    assert L.csa_page_alloc_create(4, 0, 4, ctypes.byref(h)) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_page_alloc_create(4, 2, 0, ctypes.byref(h)) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_page_alloc_create(4, 2, 4, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_page_alloc_reserve(None, 0, 1) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_page_alloc_release(None, 0) == csa.CSA_ERR_INVALID_ARG
    assert not L.csa_page_alloc_table(None)
    assert L.csa_page_alloc_free_pages(None) == -1
    a = csa.PageAlloc(4, 2, 3)
    for b, n in ((-1, 1), (2, 1), (0, -1), (0, 4)):
        with pytest.raises(csa.CsaError) as e:
            a.reserve(b, n)
        assert e.value.status == csa.CSA_ERR_INVALID_ARG
    with pytest.raises(csa.CsaError):
        a.release(2)
    assert a.mapped(2) == -1 and a.mapped(-1) == -1
    assert csa.status_string(csa.CSA_ERR_NO_PAGES) == "CSA_ERR_NO_PAGES"


@pytest.mark.parametrize("m,rows", [(4, 32), (128, 1), (4, 128)])
def test_pages_needed_at_block_boundaries(m, rows):
    block = m * rows  # raw tokens per page
    for n_tok in sorted({0, 1, m - 1, m, block - 1, block, block + m - 1, block + m,
                         5 * block - 1, 5 * block, 5 * block + 3 * m, 1 << 20}):
        want = -(-(n_tok // m) // rows)
        assert csa.state_pages_needed(m, rows, n_tok) == want, (m, rows, n_tok)
    assert csa.state_pages_needed(0, rows, 10) == -1
    assert csa.state_pages_needed(m, 0, 10) == -1
    assert csa.state_pages_needed(m, rows, -1) == -1


@pytest.mark.parametrize("n_pages", [40, 14], ids=["enough_pages", "runs_out"])
def test_a_decode_loop_gets_the_oracle_page_tables(n_pages):
    m, rows, c, B = 4, 2, 8, 3
    pool = SC.PagePool(n_pages, rows, c)
    alloc = csa.PageAlloc(n_pages, B, 16)
    g = np.random.default_rng(5)
    bias = g.standard_normal((2 * m, c))

    def new_request():
        return SC.CsaState(pool, m=m, c=c, bias=bias, n_win=0, r=2, base=10000.0, eps=1e-6,
                           block_tokens=m * rows)

    live = [new_request() for _ in range(B)]
    lengths = [37, 23, 51]  # tokens before a request finishes and a new one takes its row
    done, ran_out = 0, False
    for step in range(600):
        b = step % B
        st = live[b]
        if st.n_tok == lengths[b]:  # finished: pages back to the pool, a new request starts
            st.release()
            alloc.release(b)
            live[b] = st = new_request()
            lengths[b] = int(g.integers(10, 60))
            done += 1
        need = csa.state_pages_needed(m, rows, st.n_tok + 1)
        try:
            alloc.reserve(b, need)
        except csa.CsaError as e:
            assert e.status == csa.CSA_ERR_NO_PAGES
            with pytest.raises(MemoryError):  # the oracle runs out at the same token
                st.append(*g.standard_normal((5, c)))
            ran_out = True
            break
        st.append(*g.standard_normal((5, c)))
        for bb, s in enumerate(live):
            assert alloc.table[bb, :len(s.page_table)].tolist() == s.page_table, (step, bb)
            assert (alloc.table[bb, len(s.page_table):] == -1).all()
        assert alloc.free_pages == len(pool.free)
    assert ran_out == (n_pages == 14)
    if not ran_out:
        assert done >= 10  # many requests finished and gave their pages back
