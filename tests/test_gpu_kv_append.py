"""Block commit into the paged context cache (tt_kv_append, the context update of Algorithm 1) against the
oracle's append_block: the gathered context after the append is bit-exact the old context
followed by the block; the pages taken are the top of the free stack; the device reports a
sequence it cannot give pages; attention over the grown cache matches the oracle."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api
from denoiser_attention_b200 import binding as B
from oracle import tt_oracle as O
from tests._parity import assert_close_attn, np64

pytestmark = pytest.mark.gpu


def _pool(lens, S, Hkv, d, dtype, page_size, num_pages, max_pages, seed):
    """A paged pool holding each sequence's existing context in seeded pages, and a free stack of
    the pages nobody uses (shuffled)."""
    g = torch.Generator().manual_seed(seed)
    Bn = len(lens)
    k_ctx = torch.randn((num_pages, page_size, Hkv, d), generator=g).to(dtype)
    v_ctx = torch.randn((num_pages, page_size, Hkv, d), generator=g).to(dtype)
    order = torch.randperm(num_pages, generator=g).tolist()
    table = torch.full((Bn, max_pages), -1, dtype=torch.int32)
    used = 0
    for b, L in enumerate(lens):
        for i in range((L + page_size - 1) // page_size):
            table[b, i] = order[used]
            used += 1
    free = torch.tensor(order[used:], dtype=torch.int32)
    k_new = torch.randn((Bn, S, Hkv, d), generator=g).to(dtype)
    v_new = torch.randn((Bn, S, Hkv, d), generator=g).to(dtype)
    return k_ctx, v_ctx, table, free, k_new, v_new


def _run(k_ctx, v_ctx, table, free, k_new, v_new, lens):
    dev = "cuda"
    t = {n: x.to(dev) for n, x in dict(k_ctx=k_ctx, v_ctx=v_ctx, table=table, free=free, k_new=k_new,
                                        v_new=v_new).items()}
    t["lens"] = torch.tensor(lens, dtype=torch.int32, device=dev)
    t["count"] = torch.tensor([free.numel()], dtype=torch.int32, device=dev)
    ws = api.append_block_kv(t["k_new"], t["v_new"], t["k_ctx"], t["v_ctx"], t["table"], t["lens"], t["free"],
                             t["count"])
    st, detail = B.tt_get_device_error(ws)
    torch.cuda.synchronize()
    return t, st, detail


@pytest.mark.parametrize("dtype,page_size,lens,S", [
    (torch.bfloat16, 256, [0, 4096, 300, 511, 5000, 256], 16),
    (torch.bfloat16, 128, [127, 128, 1, 0], 16),
    (torch.float32, 16, [15, 16, 3, 40], 8),
    (torch.bfloat16, 16, [10, 33], 64),      # a block spanning several new pages
])
def test_append_matches_oracle(cuda_lib, dtype, page_size, lens, S):
    Hkv, d = 2, 128 if dtype == torch.bfloat16 else 64
    num_pages = sum((L + S + page_size - 1) // page_size for L in lens) + 7
    max_pages = max((L + S + page_size - 1) // page_size for L in lens) + 1
    k_ctx, v_ctx, table, free, k_new, v_new = _pool(lens, S, Hkv, d, dtype, page_size, num_pages, max_pages, seed=S)
    t, st, _ = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)
    assert st == B.TT_OK
    new_lens = t["lens"].cpu().tolist()
    assert new_lens == [L + S for L in lens]
    # content: gathered through the updated page table, bit-exact the oracle's concatenation
    old_k, old_v = O.gather_context(np64(k_ctx), np64(v_ctx), lens, table.numpy(), page_size)
    want_k, want_v, want_lens = O.append_block(old_k, old_v, np64(k_new), np64(v_new))
    got_k, got_v = O.gather_context(np64(t["k_ctx"]), np64(t["v_ctx"]), new_lens, t["table"].cpu().numpy(), page_size)
    assert want_lens == new_lens
    for b in range(len(lens)):
        np.testing.assert_array_equal(got_k[b], want_k[b])
        np.testing.assert_array_equal(got_v[b], want_v[b])
    # pages: the new ones are exactly the top of the free stack, distinct, and were free
    n_new = sum((L + S + page_size - 1) // page_size - (L + page_size - 1) // page_size for L in lens)
    count = int(t["count"].item())
    assert count == free.numel() - n_new
    taken = set(free[count:].tolist())
    tab = t["table"].cpu()
    new_ids = []
    for b, L in enumerate(lens):
        have = (L + page_size - 1) // page_size
        need = (L + S + page_size - 1) // page_size
        assert tab[b, :have].tolist() == table[b, :have].tolist()   # existing pages kept
        new_ids += tab[b, have:need].tolist()
    assert sorted(new_ids) == sorted(taken) and len(set(new_ids)) == len(new_ids)


def test_out_of_pages_is_reported(cuda_lib):
    lens, S, page_size = [0, 0, 0], 16, 16
    k_ctx, v_ctx, table, free, k_new, v_new = _pool(lens, S, 1, 64, torch.float32, page_size, 2, 4, seed=5)
    t, st, detail = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)   # 3 sequences, 2 free pages
    assert st == B.TT_ERR_DEVICE and detail == 4
    got = t["lens"].cpu().tolist()
    assert sorted(got) == [0, 16, 16]            # exactly the sequences that got a page advanced
    assert int(t["count"].item()) == 0


def test_page_table_full_is_reported(cuda_lib):
    lens, S, page_size = [30, 0], 16, 16         # sequence 0 would need 3 pages, the table has 2
    k_ctx, v_ctx, table, free, k_new, v_new = _pool(lens, S, 1, 64, torch.float32, page_size, 8, 2, seed=6)
    t, st, detail = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)
    assert st == B.TT_ERR_DEVICE and detail == 5
    assert t["lens"].cpu().tolist() == [30, 16]


def test_attention_over_the_grown_cache(cuda_lib):
    # Algorithm 1: block b is committed (its context KV appended); block b+1's queries then attend
    # to the grown context and their own block
    Bn, S, Hq, Hkv, d, page_size = 2, 16, 32, 2, 128, 256
    lens = [700, 1024]
    num_pages, max_pages = 16, 8
    k_ctx, v_ctx, table, free, k_new, v_new = _pool(lens, S, Hkv, d, torch.bfloat16, page_size, num_pages, max_pages,
                                                    seed=9)
    t, st, _ = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)
    assert st == B.TT_OK
    g = torch.Generator().manual_seed(10)
    q = (torch.randn((Bn, S, Hq, d), generator=g) / d ** 0.5).to(torch.bfloat16)
    kb = torch.randn((Bn, S, Hkv, d), generator=g).to(torch.bfloat16)
    vb = torch.randn((Bn, S, Hkv, d), generator=g).to(torch.bfloat16)
    out = api.denoise_attention(q.cuda(), kb.cuda(), vb.cuda(), t["k_ctx"], t["v_ctx"], t["lens"],
                                page_table=t["table"], page_size=page_size)
    torch.cuda.synchronize()
    old_k, old_v = O.gather_context(np64(k_ctx), np64(v_ctx), lens, table.numpy(), page_size)
    ck, cv, new_lens = O.append_block(old_k, old_v, np64(k_new), np64(v_new))
    stride = max(new_lens)
    ks = np.zeros((Bn, stride, Hkv, d)); vs = np.zeros((Bn, stride, Hkv, d))
    for b in range(Bn):
        ks[b, :new_lens[b]], vs[b, :new_lens[b]] = ck[b], cv[b]
    want = O.denoise_attention(np64(q), np64(kb), np64(vb), ks, vs, new_lens)
    assert_close_attn(out.cpu(), want, torch.bfloat16, "grown cache")


@pytest.mark.parametrize("trial", range(4))
def test_concurrent_out_of_pages_keeps_the_stack_consistent(cuda_lib, trial):
    # 96 sequences claim 1 or 2 pages each from a stack holding far fewer than they need, in one
    # launch: the sequences that advance hold distinct pages, exactly the top of the stack; the
    # count says how many entries are left; the sequences that fail are untouched
    rs = np.random.default_rng(50 + trial)
    Bn, S, page_size, Hkv, d = 96, 16, 16, 1, 64
    lens = [int(x) for x in rs.integers(0, 64, Bn)]
    have = [(L + page_size - 1) // page_size for L in lens]
    need = [(L + S + page_size - 1) // page_size - h for L, h in zip(lens, have)]
    max_pages = max(h + n for h, n in zip(have, need)) + 1
    n_free = sum(need) // 3
    num_pages = sum(have) + n_free + 5
    k_ctx, v_ctx, table, _, k_new, v_new = _pool(lens, S, Hkv, d, torch.float32, page_size, num_pages, max_pages,
                                                 seed=60 + trial)
    used = set(table[table >= 0].tolist())
    free = torch.tensor([p for p in rs.permutation(num_pages).tolist() if p not in used][:n_free],
                        dtype=torch.int32)
    t, st, detail = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)
    assert st == B.TT_ERR_DEVICE and detail == 4
    new_lens = t["lens"].cpu().tolist()
    tab = t["table"].cpu()
    count = int(t["count"].item())
    ok = [nl == L + S for nl, L in zip(new_lens, lens)]
    assert all(nl in (L, L + S) for nl, L in zip(new_lens, lens))
    assert any(ok) and not all(ok)
    claimed = []
    for b in range(Bn):
        assert tab[b, :have[b]].tolist() == table[b, :have[b]].tolist()
        if ok[b]:
            claimed += tab[b, have[b]:have[b] + need[b]].tolist()
        else:
            assert tab[b].tolist() == table[b].tolist()        # a failed sequence keeps its row
    assert len(set(claimed)) == len(claimed)                    # no page handed out twice
    assert count == n_free - len(claimed)                       # the count matches what was taken
    assert sorted(claimed) == sorted(free[count:].tolist())     # exactly the top of the stack
    assert not (set(claimed) & used)
    # content of the sequences that advanced
    old_k, old_v = O.gather_context(np64(k_ctx), np64(v_ctx), lens, table.numpy(), page_size)
    want_k, want_v, _ = O.append_block(old_k, old_v, np64(k_new), np64(v_new))
    got_k, got_v = O.gather_context(np64(t["k_ctx"]), np64(t["v_ctx"]), new_lens, tab.numpy(), page_size)
    for b in range(Bn):
        if ok[b]:
            np.testing.assert_array_equal(got_k[b], want_k[b])
            np.testing.assert_array_equal(got_v[b], want_v[b])


def test_bad_page_id_in_the_stack_changes_nothing(cuda_lib):
    lens, S, page_size = [0, 16], 16, 16
    k_ctx, v_ctx, table, free, k_new, v_new = _pool(lens, S, 1, 64, torch.float32, page_size, 6, 4, seed=7)
    free = torch.tensor([free[0].item(), 99], dtype=torch.int32)       # the top entry is not a page id
    t, st, detail = _run(k_ctx, v_ctx, table, free, k_new, v_new, lens)
    assert st == B.TT_ERR_DEVICE and detail == 1
    assert int(t["count"].item()) == 2
    assert t["lens"].cpu().tolist() == lens
    assert torch.equal(t["table"].cpu(), table)
