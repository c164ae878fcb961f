"""How forward_host cuts a dense batch into contiguous pieces (host logic only)."""
import pytest

from linear_recurrent_lm_wkv7_b200 import host_pieces


@pytest.mark.parametrize("B,T,parts,t_parts", [(4, 1024, 4, 1), (3, 130, 2, 1), (3, 130, 2, 3), (4, 1024, 4, 4),
                                               (1, 64, 4, 4), (2, 1000, 8, 4), (5, 7, 2, 1), (2, 0, 2, 1),
                                               (2, 0, 2, 3)])
def test_pieces_cover_every_token_once(B, T, parts, t_parts):
    groups, bounds = host_pieces(B, T, parts, t_parts)
    assert bounds[0] == 0 and bounds[-1] == T and bounds == sorted(bounds)
    assert all(b % 64 == 0 for b in bounds[:-1])  # ranges start on chunk boundaries
    seen = set()
    for b0, b1 in groups:
        for b in range(b0, b1):
            for t in range(T):
                assert (b, t) not in seen
                seen.add((b, t))
    assert len(seen) == B * T
    assert sum(b1 - b0 for b0, b1 in groups) == B
    if len(bounds) > 2:
        # token ranges: single-sequence groups, so every piece is contiguous
        assert all(b1 - b0 == 1 for b0, b1 in groups)
    else:
        assert len(groups) == min(parts, B)
    if T == 0:
        assert bounds == [0, 0]
