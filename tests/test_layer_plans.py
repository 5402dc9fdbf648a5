"""Host logic of the layers' recorded call plans (no GPU): a plan is reused only for a call whose
X and Y buffers (pointer, shape, strides, dtype) and stream all match the call that recorded it,
and the table stays bounded."""
import torch

from bit_w4a4_diffusion_smooth_b200.layer import _Plans


def _key(X, Y, s=0):
    return _Plans.key(X, Y, s)


def test_key_separates_every_checked_property():
    base = torch.zeros((64, 512), dtype=torch.bfloat16)
    Y = torch.zeros((64, 256), dtype=torch.bfloat16)
    k = _key(base, Y)
    assert k == _key(base, Y)                                            # the same buffers: a hit
    assert k != _key(base[:63], Y)                                       # fewer rows, same pointer
    assert k != _key(base[1:], Y)                                        # another pointer
    assert k != _key(torch.zeros((64, 1024), dtype=torch.bfloat16)[:, :512], Y)   # another row stride
    assert k != _key(base.view(torch.float16), Y)                        # another dtype
    assert k != _key(base, Y, s=7)                                       # another stream
    assert k != _key(base, torch.zeros((64, 256), dtype=torch.bfloat16))  # another output buffer
    Yw = torch.zeros((64, 512), dtype=torch.bfloat16)
    assert k != _key(base, Yw[:, :256])                                  # output with a wider row stride


def test_table_is_bounded_and_returns_what_was_stored():
    t = _Plans()
    for i in range(_Plans.LIMIT):
        t.put(i, ("plan", i))
    assert t.get(0) == ("plan", 0) and t.get(_Plans.LIMIT - 1) == ("plan", _Plans.LIMIT - 1)
    t.put("next", ("plan", "next"))                                      # a full table is cleared first
    assert t.get(0) is None and t.get("next") == ("plan", "next")
    assert len(t._t) == 1
