"""GPU parity of the paged cache append (sia_cache_append) against the oracle: every written code
and scale bit for bit, every other row untouched, in each index-key format (bf16 copy, per-token
power-of-two FP8, MXFP8 groups of 32) and each main-cache format (bf16 copy, FP8 with one scale
per 128-element block)."""
import numpy as np
import pytest
import torch

import indexed_sparse_attention_paged_b200 as sia
import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(seed, B=5, J=2, D=128, DC=576, P=16, extra_pages=3):
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(J, 6 * P, (B,), generator=g, dtype=torch.int32)
    pages = [(int(l) + P - 1) // P for l in lens]
    num_pages = sum(pages) + extra_pages
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    pt = torch.full((B, max(pages)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        pt[b, :n] = perm[off:off + n]
        off += n
    # magnitudes spread over many binades per token and per block, plus exact zeros and ties
    mag_k = torch.pow(2.0, torch.randint(-12, 12, (B, J, D // 32, 1), generator=g).float())
    new_k = (torch.randn((B, J, D // 32, 32), generator=g) * mag_k).reshape(B, J, D)
    new_k[0, 0, :32] = 0.0                                  # an all-zero MX group
    mag_v = torch.pow(2.0, torch.randint(-10, 10, (B, J, (DC + 127) // 128, 1), generator=g).float())
    v = torch.randn((B, J, (DC + 127) // 128, 128), generator=g) * mag_v
    new_kv = v.reshape(B, J, -1)[:, :, :DC].contiguous()
    new_kv[1, J - 1, 128:256] = 0.0                         # an all-zero main-cache block
    if B > 2:
        new_k[2, 0] = 0.0                                   # an all-zero key
    return pt, lens, new_k.to(torch.bfloat16), new_kv.to(torch.bfloat16), num_pages


@pytest.mark.parametrize("key_format", ["bf16", "fp8", "mx"])
@pytest.mark.parametrize("kv_fp8", [False, True])
def test_cache_append_matches_the_oracle_bit_for_bit(key_format, kv_fp8):
    pt, sl, new_k, new_kv, num_pages = _case(700 + 10 * ["bf16", "fp8", "mx"].index(key_format) + kv_fp8)
    B, J, D = new_k.shape
    DC, P = new_kv.shape[2], 16
    g = torch.Generator().manual_seed(5)
    nblk = (DC + 127) // 128
    if key_format == "bf16":
        k0 = torch.randint(0, 1 << 16, (num_pages, P, D), generator=g, dtype=torch.int32).to(torch.uint16)
        ks0 = None
    else:
        k0 = torch.randint(0, 256, (num_pages, P, D), generator=g, dtype=torch.int32).to(torch.uint8)
        ks0 = (torch.rand((num_pages, P), generator=g) if key_format == "fp8" else
               torch.randint(0, 255, (num_pages, P, D // 32), generator=g, dtype=torch.int32).to(torch.uint8))
    if kv_fp8:
        v0 = torch.randint(0, 256, (num_pages, P, DC), generator=g, dtype=torch.int32).to(torch.uint8)
        vs0 = torch.rand((num_pages, P, nblk), generator=g)
    else:
        v0 = torch.randint(0, 1 << 16, (num_pages, P, DC), generator=g, dtype=torch.int32).to(torch.uint16)
        vs0 = None

    # oracle on host copies
    ok, oks = k0.numpy().copy(), None if ks0 is None else ks0.numpy().copy()
    ov, ovs = v0.numpy().copy(), None if vs0 is None else vs0.numpy().copy()
    st = oracle.cache_append(new_k, new_kv, pt.numpy(), sl.numpy(), ok, ov, page_size=P,
                             k_mode=key_format, k_scale=oks, kv_scale=ovs)
    assert st == 0

    # the CUDA path on device copies
    as_dev = lambda t, dt: None if t is None else t.to(DEV).view(dt)
    k_dt = torch.bfloat16 if key_format == "bf16" else torch.float8_e4m3fn
    kd = k0.to(DEV).view(k_dt)
    ksd = None if ks0 is None else ks0.to(DEV)
    vd = v0.to(DEV).view(torch.float8_e4m3fn if kv_fp8 else torch.bfloat16)
    vsd = None if vs0 is None else vs0.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    fmt = {"bf16": sia.SIA_KEY_BF16, "fp8": sia.SIA_KEY_FP8_POW2, "mx": sia.SIA_KEY_MXFP8}[key_format]
    sia.cache_append(new_k.to(DEV), new_kv.to(DEV), pt.to(DEV), sl.to(DEV), kd, vd, key_format=fmt,
                     k_scale=ksd, kv_scale=vsd, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    raw = lambda t: t.cpu().view(torch.uint8 if t.element_size() == 1 else torch.uint16).numpy()
    np.testing.assert_array_equal(raw(kd), ok)
    np.testing.assert_array_equal(raw(vd), ov)
    if ksd is not None:
        np.testing.assert_array_equal(ksd.cpu().numpy().view(np.uint8), oks.view(np.uint8))
    if vsd is not None:
        np.testing.assert_array_equal(vsd.cpu().numpy().view(np.uint32), ovs.view(np.uint32))


def test_cache_append_bad_page_is_skipped_and_reported():
    pt, sl, new_k, new_kv, num_pages = _case(750, B=3, J=1)
    P = 16
    p = int(sl[1]) - 1
    pt[1, p // P] = num_pages + 4                       # the new token of sequence 1 has no page
    k = torch.zeros((num_pages, P, new_k.shape[2]), dtype=torch.bfloat16, device=DEV)
    v = torch.zeros((num_pages, P, new_kv.shape[2]), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sia.cache_append(new_k.to(DEV), new_kv.to(DEV), pt.to(DEV), sl.to(DEV), k, v, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & sia.SIA_DEV_BAD_PAGE
    ok = np.zeros((num_pages, P, new_k.shape[2]), np.uint16)
    ov = np.zeros((num_pages, P, new_kv.shape[2]), np.uint16)
    pt_ok = pt.clone()
    oracle.cache_append(new_k, new_kv, pt_ok.numpy(), sl.numpy(), ok, ov, page_size=P)   # skips it too
    np.testing.assert_array_equal(k.cpu().view(torch.uint16).numpy(), ok)
    np.testing.assert_array_equal(v.cpu().view(torch.uint16).numpy(), ov)
