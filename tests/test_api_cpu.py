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


def test_default_workspaces_stay_bounded():
    api._default_ws.clear()
    keep = api._workspace_for("cuda:0", 7)
    for h in range(1000, 1100):                                 # many short-lived streams
        api._workspace_for("cuda:0", h)
        api._workspace_for("cuda:0", 7)                         # one stream stays in use
    mine = [k for k in api._default_ws if str(k[0]) == "cuda:0"]
    assert len(mine) == api._DEFAULT_WS_PER_DEVICE
    assert api._workspace_for("cuda:0", 7) is keep              # the busy stream kept its scratch
    api._workspace_for("cuda:1", 7)                             # other devices count separately
    assert len([k for k in api._default_ws if str(k[0]) == "cuda:0"]) == api._DEFAULT_WS_PER_DEVICE
    api._default_ws.clear()


def test_packed_row_bytes():
    assert api.packed_row_bytes("tq2", 4096) == 1024            # 64 B per 256 weights
    assert api.packed_row_bytes("tq1", 4096) == 16 * 52         # 52 B per 256 weights
    assert api.packed_row_bytes("tq1", 11008) == 43 * 52        # not a multiple of 16 bytes
