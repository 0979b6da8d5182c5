"""dg_kv_block_commit: bit-exact append of block K/V into the caches."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hd", [64, 128])
def test_append_exact_and_length_bump(hd):
    import canvas_denoising_denoise_b200 as dg
    n_layers, B, Hkv, C, lmax = 3, 2, 4, 256, 600
    g = torch.Generator().manual_seed(0)
    ld = (8 + 2 * Hkv) * hd
    blk = [torch.randn((B, C, ld), generator=g).to(torch.bfloat16).cuda() for _ in range(n_layers)]
    kb = [t[:, :, 8 * hd:(8 + Hkv) * hd] for t in blk]
    vb = [t[:, :, (8 + Hkv) * hd:] for t in blk]
    kc = [torch.randn((B, Hkv, lmax, hd), generator=g).to(torch.bfloat16).cuda()
          for _ in range(n_layers)]
    vc = [torch.randn((B, Hkv, lmax, hd), generator=g).to(torch.bfloat16).cuda()
          for _ in range(n_layers)]
    before_k = [t.clone() for t in kc]
    lens = torch.tensor([100, 344], dtype=torch.int32, device="cuda")
    dg.kv_block_commit(kb, vb, kc, vc, lens, n_kv_heads=Hkv, head_dim=hd)
    torch.cuda.synchronize()
    dg.check_device_errors()
    assert lens.tolist() == [356, 600]
    for l in range(n_layers):
        for b, L in enumerate([100, 344]):
            want_k = kb[l][b].reshape(C, Hkv, hd).permute(1, 0, 2)
            want_v = vb[l][b].reshape(C, Hkv, hd).permute(1, 0, 2)
            assert torch.equal(kc[l][b, :, L:L + C], want_k)
            assert torch.equal(vc[l][b, :, L:L + C], want_v)
            assert torch.equal(kc[l][b, :, :L], before_k[l][b, :, :L])
            assert torch.equal(kc[l][b, :, L + C:], before_k[l][b, :, L + C:])


def test_overflow_is_reported_not_written():
    import canvas_denoising_denoise_b200 as dg
    B, Hkv, C, hd, lmax = 1, 2, 256, 64, 300
    kb = [torch.ones((B, C, Hkv * hd), dtype=torch.bfloat16, device="cuda")]
    kc = [torch.zeros((B, Hkv, lmax, hd), dtype=torch.bfloat16, device="cuda")]
    vc = [torch.zeros((B, Hkv, lmax, hd), dtype=torch.bfloat16, device="cuda")]
    lens = torch.tensor([100], dtype=torch.int32, device="cuda")
    dg.kv_block_commit(kb, kb, kc, vc, lens, n_kv_heads=Hkv, head_dim=hd)
    with pytest.raises(dg.DgError) as e:
        dg.check_device_errors()
    assert "DEVICE_CHECK" in str(e.value)
    assert int(lens.item()) == 100 and float(kc[0].abs().sum().item()) == 0.0
