"""Host-side LRU victim choice of the KV cache manager (no GPU)."""

import pytest

from generative_recommender_sequence_b200.kv_cache import choose_victims


def test_nothing_evicted_when_the_request_fits():
    assert choose_victims({1: 5, 2: 3}, {1: 4, 2: 4}, [9], need_pages=3, free_pages=3) == []


def test_least_recently_used_first_until_enough():
    last = {10: 7, 11: 2, 12: 5, 13: 1}
    pages = {10: 3, 11: 2, 12: 4, 13: 1}
    # 13 (t=1) then 11 (t=2) then 12 (t=5): 1 + 2 + 4 = 7 >= 8 - 1
    assert choose_victims(last, pages, [10], need_pages=8, free_pages=1) == [13, 11, 12]


def test_request_users_and_empty_users_are_never_victims():
    last = {1: 1, 2: 2, 3: 3}
    pages = {1: 0, 2: 5, 3: 5}
    assert choose_victims(last, pages, [2], need_pages=5, free_pages=1) == [3]


def test_ties_break_by_user_id_and_impossible_requests_raise():
    assert choose_victims({5: 1, 4: 1}, {5: 1, 4: 1}, [], need_pages=1, free_pages=0) == [4]
    with pytest.raises(RuntimeError):
        choose_victims({1: 1}, {1: 2}, [], need_pages=10, free_pages=3)
