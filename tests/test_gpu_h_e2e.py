"""GPU: the end-to-end pipeline bench.py times (pinned host q, k, v copied in
and o, lse copied out on two copy streams beside the attention, double
buffered) delivers, for its last step, exactly what a direct call on that
step's index gives."""
import pytest
import torch

import bench
from block_sparse_attention_lvsa_b200 import inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


@pytest.mark.parametrize("name,steps", [("tiny", 5), ("wan1.3b_1x_c11", 3)])
def test_e2e_last_step_equals_direct_call(bsa, name, steps):
    wl = WORKLOADS[name]
    qkv = inputs.workload_qkv(wl, 0, device="cuda")
    frames = torch.empty((wl.T, wl.T), dtype=torch.int32, device="cuda")
    counts = torch.empty((wl.T,), dtype=torch.int32, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o = torch.empty_like(qkv[0])
    lse = torch.empty((wl.H, wl.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, wl.N, wl.H, wl.d, ix), dtype=torch.uint8,
                     device="cuda")
    host = []
    r = bench.run_e2e(bsa, wl, qkv, torch.cuda.current_stream(), frames, counts, ix, o, lse, ws, steps,
                      {ph: 0 for ph in range(wl.T_per)}, 1, host_out=host)
    ho, hl = host
    assert r["h2d_bytes_per_step"] == 3 * qkv[0].numel() * 2
    assert r["d2h_bytes_per_step"] == o.numel() * 2 + lse.numel() * 4
    # the same step through a direct call: the index of the pipeline's last step
    f2, c2, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, steps - 1, device="cuda")
    o_ref, lse_ref = bsa.blocksparse_attn_fwd(*qkv, bsa.lvsa_index(wl.T, f2, c2), scale=wl.scale)
    torch.cuda.synchronize()
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(ho, o_ref.cpu()) and torch.equal(hl, lse_ref.cpu())
