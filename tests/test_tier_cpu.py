"""The page tier's replacement policy, checked with a book-keeping-only tier (no
buffers, no copies, no GPU): LRU victims, pages of one request never evicting each
other, write-back of dirty pages, prefetch limited to released slots, statistics."""
import pytest

from linear_attention_paged_b200 import build as wa_build

wa_build.build()
from linear_attention_paged_b200 import wa  # noqa: E402


def tier(n_pages=8, n_slots=3):
    return wa.Tier(n_pages=n_pages, n_slots=n_slots, page_bytes=1 << 20)


def test_fill_then_lru_victim():
    t = tier()
    assert t.ensure([0, 1, 2]) == [0, 1, 2]            # free slots in order
    assert t.stats()["misses"] == 3
    t.ensure([0])                                      # 0 becomes most recent
    s3 = t.ensure([3])[0]
    assert s3 == 1 and t.slot_of(1) == -1              # 1 was least recently handed out
    assert t.slot_of(0) == 0 and t.slot_of(2) == 2
    st = t.stats()
    assert (st["hits"], st["misses"], st["evictions"]) == (1, 4, 1)


def test_request_never_evicts_its_own_pages():
    t = tier(n_slots=3)
    t.ensure([0, 1, 2])
    # 0 and 1 are the oldest, but both are in this request: 2 must go
    slots = t.ensure([0, 1, 5])
    assert slots[0] == 0 and slots[1] == 1 and slots[2] == 2
    assert t.slot_of(2) == -1
    # duplicates in one request map to one slot
    a = t.ensure([6, 6, 0])
    assert a[0] == a[1] and t.stats()["misses"] == 5


def test_too_many_distinct_pages_is_an_error():
    t = tier(n_slots=2)
    with pytest.raises(wa.WAError):
        t.ensure([0, 1, 2])
    t.ensure([0, 1, 1, 0])                              # two distinct pages fit
    with pytest.raises(wa.WAError):
        t.ensure([8])                                  # out of range
    with pytest.raises(wa.WAError):
        t.mark_dirty(5)                                # not resident


def test_dirty_pages_are_written_back_on_eviction_and_flush():
    t = tier(n_slots=2)
    t.ensure([0, 1])
    t.mark_dirty(0)
    t.ensure([1])
    t.ensure([2])                                       # evicts 0, which is dirty
    assert t.stats()["writebacks"] == 1 and t.slot_of(0) == -1
    t.ensure([0])                                       # evicts 1 (clean): no write-back
    assert t.stats()["writebacks"] == 1
    t.mark_dirty(0); t.mark_dirty(2)
    t.flush()
    assert t.stats()["writebacks"] == 3
    t.ensure([3]); t.ensure([4])                        # evicting flushed pages writes nothing
    assert t.stats()["writebacks"] == 3


def test_prefetch_uses_free_or_released_slots_only():
    t = tier(n_slots=3)
    assert t.prefetch([5]) == 1                         # a free slot
    t.ensure([0, 1])                                    # fills the two other slots
    assert t.prefetch([6]) == 0                         # nothing released: no victim
    t.release()
    # pages 0 and 1 were released; page 5's prefetch has not been asked for: kept
    assert t.prefetch([6, 7, 3]) == 2
    assert t.slot_of(5) == 0 and t.slot_of(6) >= 0 and t.slot_of(7) >= 0 and t.slot_of(3) == -1
    assert t.stats()["prefetches"] == 3
    assert t.ensure([6]) == [t.slot_of(6)]              # prefetched earlier: a prefetch hit
    assert t.stats()["prefetch_hits"] == 1 and t.stats()["hits"] == 0
    t.ensure([0])                                       # demand evicts the LRU slot, here page 5's
    assert t.slot_of(5) == -1


def test_create_validation():
    with pytest.raises(wa.WAError):
        wa.Tier(n_pages=0, n_slots=1, page_bytes=1)
    with pytest.raises(wa.WAError):
        wa.Tier(n_pages=4, n_slots=0, page_bytes=1)
