"""Host logic of DecodeStep's pipelined copies (no GPU needed).

The layers' input rows are copied in by chunks of growing length, and the compute waits for
a chunk only at its first layer; the outputs go back in chunks that shrink toward the last
layer.  The chunks must cover every layer exactly once, in order.
"""
import pytest

from paged_kv_cache_460_b200.step import DecodeStep


@pytest.mark.parametrize("L", [1, 2, 3, 5, 8, 21, 32, 33, 80])
def test_chunks_tile_the_layers_in_order(L):
    ch = DecodeStep._chunks(L)
    assert ch[0] == (0, 1)                          # layer 0 waits only for its own rows
    assert ch[-1][1] == L
    for (lo, hi), (lo2, hi2) in zip(ch, ch[1:]):
        assert hi == lo2 and lo < hi
    lengths = [hi - lo for lo, hi in ch]
    for a, b in zip(lengths, lengths[1:-1]):        # x4 growth, the last one cut at L
        assert b == 4 * a
    assert len(ch) <= 1 + max(0, (L - 1).bit_length() // 2 + 1)   # few waits on the compute stream


def test_output_chunks_mirror_the_input_chunks():
    L = 32
    outs = [(L - hi, L - lo) for lo, hi in reversed(DecodeStep._chunks(L))]
    assert outs[0][0] == 0 and outs[-1] == (L - 1, L)      # the last copy back is one layer
    covered = [i for lo, hi in outs for i in range(lo, hi)]
    assert covered == list(range(L))
