"""Host page bookkeeping: on-demand allocation, bounded waste, shared prefix
pages and the Eq. 2 page count (CPU only)."""
import numpy as np
import pytest

import oracle
from paged_kv_cache_466_b200 import pages
from paged_kv_cache_466_b200 import workloads as W


def test_waste_is_at_most_p_minus_one():
    alloc = pages.PageAllocator(4096)
    for T in list(range(1, 70)) + [4096, 4097, 32768 // 16 * 16 - 1]:
        r = pages.Request(alloc, 16)
        r.append(T)
        assert len(r.pages) == pages.pages_for(T, 16)
        assert 0 <= r.wasted_slots <= 15
        r.release()
    assert alloc.free_pages == 4096


def test_slots_follow_the_table():
    alloc = pages.PageAllocator(100, order=np.random.default_rng(0).permutation(100))
    r = pages.Request(alloc, 16)
    slots = r.append(50)
    for pos, page, slot in slots:
        assert page == r.pages[pos // 16] and slot == pos % 16
    t = pages.block_tables([r], max_pages=6)
    assert t.shape == (1, 6) and list(t[0, :4]) == r.pages and list(t[0, 4:]) == [-1, -1]


def test_pool_exhaustion_and_double_free():
    alloc = pages.PageAllocator(2)
    r = pages.Request(alloc, 16)
    r.append(32)
    with pytest.raises(pages.OutOfPages):
        r.append(1)
    p = r.pages[0]
    r.release()
    with pytest.raises(ValueError):
        alloc.release(p)


def test_shared_prefix_pages_and_eq2_count():
    """128 requests sharing a 125-page prefix, each with its own suffix: the
    allocator uses exactly Eq. 2's page count, 15,875 fewer than private copies."""
    shared, _ = W.prefix()
    suffix = shared.notes["suffix"]
    alloc = pages.PageAllocator(shared.num_pages)
    first = pages.Request(alloc, 16)
    first.append(2000)
    reqs = [first]
    for _ in range(len(suffix) - 1):
        r = pages.Request(alloc, 16)
        r.share_prefix(first, 2000)
        reqs.append(r)
    for r, s in zip(reqs, suffix):
        r.append(s)
    lengths = [2000 + s for s in suffix]
    assert alloc.used_pages == pages.pages_in_use(reqs) == oracle.eq2_pages_shared(lengths, 2000, 16)
    assert oracle.eq2_pages_unshared(lengths, 16) - alloc.used_pages == 15_875
    assert all(alloc.refcount(p) == 128 for p in first.pages[:125])
    with pytest.raises(ValueError):      # appending into a shared page needs copy-on-write
        r2 = pages.Request(alloc, 16)
        r2.share_prefix(first, 16)
        r2.length = 15                    # pretend the shared page is partly empty
        r2.append(1)
    for r in reqs:
        r.release()
    assert alloc.used_pages == 1          # r2's reference to the first prefix page


def test_memory_helpers_match_the_pages():
    assert pages.kv_bytes(80, 8, 128, 8192, 2) == 2_684_354_560
    assert pages.kv_bytes(32, 32, 128, 4096, 2) == 2 ** 31
    # the 70B-shaped single-layer pool: 8192 pages of 32 tokens x 8 heads x 128
    assert pages.pool_bytes(8192, 8, 32, 128) == 1_073_741_824
    assert pages.pool_bytes(10, 8, 16, 128, "u8") == 2 * 10 * 8 * 16 * 136
    assert pages.pool_bytes(10, 8, 16, 128, "fp8") == 2 * 10 * 8 * 16 * 136
    assert pages.pool_bytes(10, 8, 16, 128, "u4") == 2 * 10 * 8 * 16 * 72
    with pytest.raises(ValueError):
        pages.pool_bytes(10, 8, 16, 128, "int3")


@pytest.mark.parametrize("kind", ["bf16", "u8", "fp8", "u4"])
@pytest.mark.parametrize("shape", [(7, 2, 16, 64), (3, 8, 32, 128)])
def test_pool_bytes_is_what_a_pool_holds(kind, shape):
    # the formula against the tensors the binding actually allocates (host
    # memory here: nothing is launched)
    from paged_kv_cache_466_b200 import KVPool
    pool = KVPool(*shape, dtype=kind, device="cpu")
    assert pages.pool_bytes(*shape, kind) == sum(t.numel() * t.element_size()
                                                 for t in pool.tensors())
