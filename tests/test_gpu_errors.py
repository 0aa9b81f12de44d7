"""Error paths of the C ABI on a GPU: argument errors come back before any launch, device-found
errors (non-finite coordinates) land in the workspace status word; nothing traps."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")


def test_shape_errors():
    c = torch.zeros((100, 3), device="cuda")
    with pytest.raises(bts.BtsError) as e:
        bts.bt_build(c, 32)  # 100 is not 32 * 2^L
    assert e.value.status == "BT_ERR_SHAPE"
    with pytest.raises(bts.BtsError):
        bts.bt_build(torch.zeros((96, 3), device="cuda"), 32)
    q = torch.zeros((128, 2, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bts.BtsError) as e:
        bts.bt_ball_attention(q, q, q, None, 32)  # d = 48 unsupported
    assert e.value.status == "BT_ERR_SHAPE"


def test_workspace_too_small():
    c = torch.zeros((1024, 3), device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(bts.BtsError) as e:
        bts.bt_build(c, 32, ws=ws)
    assert e.value.status == "BT_ERR_WORKSPACE"


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_nonfinite_reported_on_device(bad):
    pts = workloads.uniform_cloud(4096, 3)
    pts[1234, 2] = bad
    ws = bts.workspace([0, 4096], 32)
    bts.bt_build(torch.from_numpy(pts).cuda(), 32, ws=ws)
    assert bts.bt_build_device_status(ws) == 3  # BT_ERR_NONFINITE
    # the context stays usable: a clean build on the same workspace reports OK
    bts.bt_build(torch.from_numpy(workloads.uniform_cloud(4096, 4)).cuda(), 32, ws=ws)
    assert bts.bt_build_device_status(ws) == 0


def test_segmented_argument_errors():
    c = torch.zeros((10, 3), device="cuda")
    for offsets in ([0, 5, 5, 10], [1, 10], [0, 11, 10]):
        with pytest.raises(bts.BtsError):
            bts.bt_build_segmented(c, offsets, 4)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(bts.BtsError) as e:
        bts.bt_build_segmented(c, list(range(0, 66)), 1, ws=ws)  # 65 clouds
    assert e.value.status == "BT_ERR_UNSUPPORTED"
