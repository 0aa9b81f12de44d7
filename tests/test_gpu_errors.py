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
    assert bts.bt_last_device_status() == 3  # the stream's word says the same, and is cleared by reading it
    # the context stays usable: a clean build on the same workspace reports OK
    bts.bt_build(torch.from_numpy(workloads.uniform_cloud(4096, 4)).cuda(), 32, ws=ws)
    assert bts.bt_build_device_status(ws) == 0
    assert bts.bt_last_device_status() == 0


@pytest.mark.parametrize("n,m,flags", [(4096, 32, 1), (65536, 128, 0), (3000, 16, 1)])
def test_nonfinite_reported_on_every_build_shape(n, m, flags):
    # narrow one-launch clusters, the record path (65,536 slots) and a padded cloud: the status word says
    # BT_ERR_NONFINITE and a clean build on the same workspace afterwards reports OK
    pts = workloads.uniform_cloud(n, 5)
    pts[n // 3, 0] = np.nan
    ws = bts.workspace([0, n], m)
    bts.bt_build_segmented_ex(torch.from_numpy(pts).cuda(), [0, n], m, flags, ws=ws)
    assert bts.bt_build_device_status(ws) == 3
    assert bts.bt_last_device_status() == 3
    bts.bt_build_segmented_ex(torch.from_numpy(workloads.uniform_cloud(n, 6)).cuda(), [0, n], m, flags, ws=ws)
    assert bts.bt_build_device_status(ws) == 0
    assert bts.bt_last_device_status() == 0


def test_segmented_argument_errors():
    c = torch.zeros((10, 3), device="cuda")
    for offsets in ([0, 5, 5, 10], [1, 10], [0, 11, 10]):
        with pytest.raises(bts.BtsError):
            bts.bt_build_segmented(c, offsets, 4)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(bts.BtsError) as e:
        bts.bt_build_segmented(c, list(range(0, 66)), 1, ws=ws)  # 65 clouds
    assert e.value.status == "BT_ERR_UNSUPPORTED"


def test_attention_perm_entry_out_of_range_is_recorded_not_read(orc):
    n, m, H, d = 256, 128, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 17)
    perm = np.arange(n, dtype=np.int32)
    perm[5] = 10 ** 6  # not a row of Q/K/V
    Q, K, V = (torch.from_numpy(t.view(np.int16)).cuda().view(torch.bfloat16) for t in (q, k, v))
    out = torch.full_like(Q, 7.0)
    bts.bt_ball_attention(Q, K, V, torch.from_numpy(perm).cuda(), m, out=out)
    assert bts.bt_last_device_status() == 8  # BT_ERR_INTERNAL, then cleared
    assert bts.bt_last_device_status() == 0
    got = out.float().cpu().numpy()
    assert np.all(got[5] == 7.0)  # the slot was treated as a dummy: row 5 is named by no valid slot
    ref_perm = perm.copy()
    ref_perm[5] = -1
    want = orc.ball_attention(q, k, v, m, ref_perm)
    keep = np.arange(n) != 5
    assert np.abs(got[keep] - want[keep]).max() <= 2e-2
