"""Host-side arithmetic of context-parallel decode (token_level_sparse_hs2_b200.cp), on CPU.

A shard [offset, offset + local_len) of a context of global_len tokens holds
local_window(...) positions of the forced window [global_len - window, global_len): checked
against counting the positions one by one, over every split of small contexts. The shard's own
selection keeps that many window positions plus its topk best candidates, so its count bound
min(local_len, topk + local window) is what cp_block_decode sizes its buffers by.
"""
import itertools

from token_level_sparse_hs2_b200 import cp


def brute_window(offset, local_len, global_len, window):
    first = max(0, global_len - window)
    return sum(1 for g in range(offset, offset + local_len) if g >= first)


def test_local_window_equals_counting_every_position():
    for global_len in (1, 5, 17, 40):
        for window in (1, 3, 16, 64):
            for a, b in itertools.combinations(range(global_len + 1), 2):
                assert cp.local_window(a, b - a, global_len, window) == \
                    brute_window(a, b - a, global_len, window), (a, b, global_len, window)


def test_shard_windows_add_up_to_the_window():
    for global_len, window in ((700, 16), (4096, 128), (100, 128)):
        for bounds in ([0, global_len], [0, global_len // 3, global_len - 5, global_len],
                       [0, 1, 2, global_len - 1, global_len]):
            total = sum(cp.local_window(bounds[i], bounds[i + 1] - bounds[i], global_len, window)
                        for i in range(len(bounds) - 1))
            assert total == min(window, global_len)
