"""The guard-band helper used by the GPU canary tests, checked on CPU: it
notices a write before, after or between the rows of a region, and none
inside the rows."""
import torch

from _canary import GUARD, PATTERN, Canary


def test_rows_inside_are_fine_padding_and_guards_are_not():
    c = Canary(6 * 40 * 2, "cpu")
    m = c.matrix(torch.bfloat16, 6, 33, 40)
    assert m.shape == (6, 33) and m.stride() == (40, 1)
    m.fill_(1.5)
    assert c.intact()
    assert c.region().view(torch.bfloat16).view(6, 40)[:, :33].eq(1.5).all()
    c.region()[33 * 2] = 0                      # first padding byte of row 0
    assert not c.intact()


def test_guards_catch_writes_just_outside():
    for where in (GUARD - 1, GUARD + 512, GUARD + 512 + GUARD - 1):
        c = Canary(512, "cpu")
        c.matrix(torch.uint8, 4, 128, 128).fill_(7)
        assert c.intact()
        c.buf[where] = PATTERN ^ 0xFF
        assert not c.intact(), where


def test_tail_past_the_last_row_is_guarded():
    c = Canary(1000, "cpu")
    c.matrix(torch.float32, 3, 64, 64).fill_(2.0)  # 768 bytes
    assert c.intact()
    c.region()[900] = 0
    assert not c.intact()


def test_zeroed_workspace_is_all_writable():
    c = Canary(2048, "cpu")
    ws = c.zeroed()
    assert ws.eq(0).all() and c.intact()
    ws[-1] = 3
    assert c.intact()
    c.buf[GUARD + 2048] = 0
    assert not c.intact()
    assert c.ptr() - c.buf.data_ptr() == GUARD and GUARD % 256 == 0
