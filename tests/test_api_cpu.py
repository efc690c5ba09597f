"""Host-side behaviour of the torch wrappers that needs no device."""
import bit_mixed_precision_tri_b200.api as api


def test_default_workspace_per_device_and_stream():
    a = api._workspace_for("cuda:0", 0)
    assert api._workspace_for("cuda:0", 0) is a                 # same stream: reused
    b = api._workspace_for("cuda:0", 0x1234)
    assert b is not a                                           # another stream: its own scratch
    c = api._workspace_for("cuda:1", 0)
    assert c is not a and str(c.device) == "cuda:1"             # another device
    assert a.buf is None                                        # nothing allocated until a call


def test_packed_row_bytes():
    assert api.packed_row_bytes("tq2", 4096) == 1024            # 64 B per 256 weights
    assert api.packed_row_bytes("tq1", 4096) == 16 * 52         # 52 B per 256 weights
    assert api.packed_row_bytes("tq1", 11008) == 43 * 52        # not a multiple of 16 bytes
