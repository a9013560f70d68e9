"""Host logic of the stack runner, on the CPU: the chunks in which the
end-to-end step copies inputs up and outputs down.  Every layer's input must
go up in exactly one chunk that has landed no later than its first product
needs it (the chunks grow slowly enough), and every layer's output must come
down in exactly one chunk whose copy follows the chunk's last layer."""
import types

import pytest

from gemm_exl3_gemv_b200.stack import Stack


def _fake(n):
    fake = types.SimpleNamespace(layers=list(range(n)))
    fake._copy_chunks = lambda: Stack._copy_chunks(fake)
    return fake


def _chunks(n):
    return Stack._copy_chunks(_fake(n))


@pytest.mark.parametrize("n", [1, 2, 3, 5, 16, 64, 100])
def test_input_chunks_cover_every_layer_once_and_grow_slowly(n):
    ch = _chunks(n)
    assert ch[0] == (0, 1)
    assert [x for a, b in ch for x in range(a, b)] == list(range(n))
    # the copy of chunk [a, b) starts after the copies of layers < a and takes
    # about (b - a) half-layers; the products reach layer a after a layers:
    # the chunk has landed in time while b <= 2 a + 1
    for a, b in ch[1:]:
        assert b <= 2 * a + 1, (a, b)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 16, 64, 100])
def test_output_chunks_mirror_the_input_chunks(n):
    out = Stack._out_chunks(_fake(n))
    covered = []
    for li in range(n):
        if li in out:
            a, b = out[li]
            assert b - 1 == li                                # copied once its last layer is done
            covered += list(range(a, b))
    assert covered == list(range(n))
    assert out[n - 1] == (n - 1, n)                           # the last layer's output alone
