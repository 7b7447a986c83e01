"""Shared-prefix pages on the GPU: decode through block tables that share
prefix pages, and the copy-on-write append of a shared boundary page, against
the oracle."""
import numpy as np
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from tests.gpu_util import log_error, np64

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.detach().cpu()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).numpy()


def _shared_pool(B, Hkv, D, P, prefix, private, dtype, gen):
    """Pool with `prefix` tokens shared by every sequence (the boundary page of
    the prefix included when prefix % P != 0) and `private[b]` more pages per
    sequence; returns (k, v, block_table, boundary page id or -1)."""
    n_shared = (prefix + P - 1) // P
    n_priv = max(private)
    n_pages = n_shared + B * n_priv
    k = torch.randn((n_pages, Hkv, P, D), generator=gen).to(dtype)
    v = torch.randn((n_pages, Hkv, P, D), generator=gen).to(dtype)
    perm = torch.randperm(n_pages, generator=gen).to(torch.int32)
    bt = torch.full((B, n_shared + n_priv), -1, dtype=torch.int32)
    for b in range(B):
        bt[b, :n_shared] = perm[:n_shared]
        bt[b, n_shared:n_shared + private[b]] = perm[n_shared + b * n_priv:n_shared + b * n_priv + private[b]]
    boundary = int(perm[n_shared - 1]) if prefix % P else -1
    return k, v, bt, boundary


@pytest.mark.parametrize("dtype,Hq,Hkv,T", [(torch.bfloat16, 64, 8, 1), (torch.float32, 8, 2, 2),
                                             (torch.bfloat16, 32, 8, 3)])
def test_copy_on_write_append_then_decode(dtype, Hq, Hkv, T):
    gen = torch.Generator().manual_seed(11)
    B, D, P, prefix = 4, 128 if dtype == torch.bfloat16 else 64, 16, 1000   # 1000 % 16 = 8
    k, v, bt, boundary = _shared_pool(B, Hkv, D, P, prefix, [3, 3, 3, 3], dtype, gen)
    n_shared = (prefix + P - 1) // P
    # every sequence has exactly the shared prefix; its boundary entry gets a
    # fresh page (the first private one), the old boundary page is the source
    bt2 = bt.clone()
    for b in range(B):
        bt2[b, n_shared - 1] = bt[b, n_shared]
        bt2[b, n_shared] = bt[b, n_shared + 1]
        bt2[b, n_shared + 1] = bt[b, n_shared + 2]
        bt2[b, n_shared + 2] = -1
    seq = torch.full((B,), prefix, dtype=torch.int32)
    cow = torch.full((B,), boundary, dtype=torch.int32)
    q = torch.randn((B, T, Hq, D), generator=gen).to(dtype)
    kn = torch.randn((B, T, Hkv, D), generator=gen).to(dtype)
    vn = torch.randn((B, T, Hkv, D), generator=gen).to(dtype)
    sdt = "f32" if dtype == torch.float32 else "bf16"
    q_rot, kc, vc = oracle.append_rope(np64(q), np64(kn), np64(vn), np64(k), np64(v), seq.numpy(),
                                       10000.0, sdt, bt2.numpy(), cow_src=cow.numpy())
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvd.append_rope_cow(dq, kn.cuda(), vn.cuda(), dk, dv, seq.cuda(), bt2.cuda(), cow.cuda(),
                        status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    gk, gv = dk.cpu(), dv.cpu()
    # the shared pages are untouched, the copied slots are bit for bit the source's
    for j in range(n_shared):
        assert np.array_equal(_bits(gk[bt[0, j]]), _bits(k[bt[0, j]]))
    for b in range(B):
        fresh = int(bt2[b, n_shared - 1])
        assert np.array_equal(_bits(gk[fresh, :, :prefix % P]), _bits(k[boundary, :, :prefix % P]))
        assert np.array_equal(_bits(gv[fresh, :, :prefix % P]), _bits(v[boundary, :, :prefix % P]))
    # new k within one storage ulp of the oracle, v bit for bit
    np.testing.assert_allclose(np64(gk), kc, rtol=2.0 ** -7, atol=0)
    assert np.array_equal(np64(gv), vc)
    out = kvd.decode_attention_paged(dq, dk, dv, seq.cuda(), bt2.cuda(), scale=D ** -0.5,
                                     max_kv_len=prefix + T, out_dtype=torch.float32)
    ref = oracle.decode_attention(q_rot, kc, vc, seq.numpy(), D ** -0.5, bt2.numpy())
    err = oracle.max_abs_diff(np64(out), ref)
    log_error(f"cow[{sdt},{Hq}/{Hkv},T{T}]", err)
    assert err <= (1e-5 if dtype == torch.float32 else 2e-3)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (64, 8)])
def test_shared_prefix_decode(Hq, Hkv):
    """64 sequences with a 2048-token shared prefix and private suffixes."""
    gen = torch.Generator().manual_seed(12)
    B, D, P, prefix = 64, 128, 16, 2048
    priv = [int(x) for x in torch.randint(1, 20, (B,), generator=gen)]
    k, v, bt, _ = _shared_pool(B, Hkv, D, P, prefix, priv, torch.bfloat16, gen)
    seq = torch.tensor([prefix + 16 * n - 1 for n in priv], dtype=torch.int32)
    q = torch.randn((B, 1, Hq, D), generator=gen).to(torch.bfloat16)
    out = kvd.decode_attention_paged(q.cuda(), k.cuda(), v.cuda(), seq.cuda(), bt.cuda(),
                                     scale=D ** -0.5, max_kv_len=int(seq.max()) + 1,
                                     out_dtype=torch.float32)
    ref = oracle.decode_attention(np64(q), np64(k), np64(v), seq.numpy(), D ** -0.5, bt.numpy())
    err = oracle.max_abs_diff(np64(out), ref)
    log_error(f"shared_prefix[{Hq}/{Hkv}]", err)
    assert err <= 2e-3


@pytest.mark.parametrize("dtype,Hq,Hkv,T,B", [(torch.bfloat16, 64, 8, 1, 12), (torch.float32, 8, 2, 2, 6),
                                               (torch.bfloat16, 32, 8, 3, 8)])
def test_cascade_decode_matches_plain_and_oracle(dtype, Hq, Hkv, T, B):
    """Prefix once per group of sequences + suffix per sequence + merge equals
    the plain paged decode and the oracle."""
    from kv_cache_decode_rope_b200.prefix import cascade_decode
    gen = torch.Generator().manual_seed(13)
    D = 128 if dtype == torch.bfloat16 else 64
    P, prefix = 16, 1024
    priv = [int(x) for x in torch.randint(1, 12, (B,), generator=gen)]
    k, v, bt, _ = _shared_pool(B, Hkv, D, P, prefix, priv, dtype, gen)
    # lengths: the prefix plus up to the private capacity (a few tokens short of it)
    seq = torch.tensor([prefix + 16 * n - T - (b % 3) for b, n in enumerate(priv)], dtype=torch.int32)
    q = torch.randn((B, T, Hq, D), generator=gen).to(dtype)
    dq, dk, dv, dbt, dseq = q.cuda(), k.cuda(), v.cuda(), bt.cuda(), seq.cuda()
    got = cascade_decode(dq, dk, dv, dseq, dbt, prefix, scale=D ** -0.5, out_dtype=torch.float32)
    plain = kvd.decode_attention_paged(dq, dk, dv, dseq, dbt, scale=D ** -0.5,
                                       max_kv_len=int(seq.max()) + T, out_dtype=torch.float32)
    ref = oracle.decode_attention(np64(q), np64(k), np64(v), seq.numpy(), D ** -0.5, bt.numpy())
    torch.cuda.synchronize()
    err = oracle.max_abs_diff(np64(got), ref)
    log_error(f"cascade[{Hq}/{Hkv},T{T},B{B}]", err)
    tol = 1e-5 if dtype == torch.float32 else 2e-3
    assert err <= tol
    assert oracle.max_abs_diff(np64(got), np64(plain)) <= tol
