"""GPU parity of sd_commit against the oracle (integer closed form, bit-exact)."""
import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import commit as OC
from tests.gpu_util import DEV, status_ok, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hidden_dtype", ["bf16", "f32"])
def test_commit_matches_oracle_and_poisons(hidden_dtype):
    B, k, bs, d, hkv, D = 64, 3, 16, 96, 2, 64
    rng = np.random.default_rng(0)
    L = S.ctx_lengths(1, B, 0, 300)
    table, nb = S.block_table(2, L, k + 1, bs, shuffle=True)
    a = rng.integers(0, k + 1, B).astype(np.int32)
    if hidden_dtype == "bf16":
        hidden = S.bf16(S.normal(3, (B, k + 1, d)))
        hd = sd.SD_BF16
    else:
        hidden = torch.from_numpy(S.normal(3, (B, k + 1, d)))
        hd = sd.SD_F32
    cache = torch.zeros((nb, hkv, bs, D), dtype=torch.bfloat16, device=DEV)
    ctx = to_dev(torch.from_numpy(L))
    slots = torch.full((B, k + 1), -9, dtype=torch.int32, device=DEV)
    nh = torch.empty((B, d), dtype=hidden.dtype, device=DEV)
    plist = sd.poison_list([(cache, hkv, D, sd.SD_BF16)])
    desc = sd.CommitDesc(batch=B, k=k, block_size=bs, max_blocks_per_seq=table.shape[1],
                         num_blocks=nb, d=d, hidden_dtype=hd, n_poison=1, poison=plist)
    sd.sd_commit(desc, to_dev(torch.from_numpy(table)), ctx, to_dev(torch.from_numpy(a)), slots,
                 to_dev(hidden), nh)
    torch.cuda.synchronize()
    ref = OC.commit(L, a, table, bs, k + 1, hidden.float().numpy())
    assert np.array_equal(ctx.cpu().numpy(), ref["ctx_len"])
    assert np.array_equal(slots.cpu().numpy(), ref["committed_slots"])
    assert torch.equal(nh.cpu().float(), torch.from_numpy(ref["next_hidden"]).float())
    c = cache.cpu().float()
    rolled = {(s // bs, s % bs) for (_, _, s) in ref["rolled_back"]}
    for (blk, row) in rolled:
        assert torch.isnan(c[blk, :, row]).all()
    nan_rows = torch.isnan(c).all(dim=-1).any(dim=1).nonzero().tolist()
    assert {(b_, r_) for b_, r_ in nan_rows} == rolled
    assert status_ok()


def test_commit_flags_out_of_range_accept_count():
    B, k, bs = 2, 2, 16
    table = torch.arange(2, dtype=torch.int32).reshape(2, 1)
    ctx = torch.tensor([3, 4], dtype=torch.int32, device=DEV)
    a = torch.tensor([1, 5], dtype=torch.int32, device=DEV)  # 5 > k
    slots = torch.full((B, k + 1), -9, dtype=torch.int32, device=DEV)
    desc = sd.CommitDesc(batch=B, k=k, block_size=bs, max_blocks_per_seq=1, num_blocks=2)
    sd.sd_commit(desc, to_dev(table), ctx, a, slots)
    torch.cuda.synchronize()
    assert ctx.cpu().tolist() == [5, 4]  # the bad sequence is left untouched
    assert sd.sd_device_status_read() == sd.SD_ERR_DEVICE
    sd.sd_device_status_clear()
    assert status_ok()


def test_commit_advances_step_counter():
    B, k, bs = 4, 2, 16
    L = np.array([5, 17, 0, 40], np.int32)
    table, nb = S.block_table(0, L, 4 * (k + 1), bs, shuffle=False)
    counter = torch.tensor([41], dtype=torch.int64, device=DEV)
    ctx = to_dev(torch.from_numpy(L))
    a = torch.tensor([0, 2, 1, 2], dtype=torch.int32, device=DEV)
    slots = torch.empty((B, k + 1), dtype=torch.int32, device=DEV)
    desc = sd.CommitDesc(batch=B, k=k, block_size=bs, max_blocks_per_seq=table.shape[1],
                         num_blocks=nb, step_ptr=counter.data_ptr())
    for _ in range(3):
        sd.sd_commit(desc, to_dev(torch.from_numpy(table)), ctx, a, slots)
    torch.cuda.synchronize()
    assert counter.item() == 44
    assert ctx.cpu().tolist() == [5 + 3, 17 + 9, 0 + 6, 40 + 9]
    assert status_ok()
