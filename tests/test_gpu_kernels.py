"""GPU parity of the single-step kernels (through the C ABI) against the CPU oracle.

Bars: indices/masks/gathers bit-exact; fp32 scores within 1e-3 relative; bf16
scores within 2e-2 relative; GEMM against an fp32 PyTorch reference."""
import numpy as np
import pytest
import torch

import synth
from oracle import movement as omv
from oracle import predictor as opr
from oracle import scores as osc
from oracle import select as osel
from oracle.bf16 import from_bits
from tests.layer_harness import bits_to_torch, rel_max, torch_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import token_sparse_long_b200 as J
    from token_sparse_long_b200 import api
    J._lib.load()
    J._api_test_exp2 = api.jenga_test_exp2
    return J


# ------------------------------------------------------------------ tcgen05 GEMM
@pytest.mark.parametrize("M,N,K,bn", [(128, 256, 64, 256), (200, 512, 128, 256), (384, 768, 1024, 256),
                                      (130, 32, 4096, 32), (1000, 1024, 4096, 256)])
def test_gemm_against_fp32_matmul(J, M, N, K, bn):
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    a = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    b = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    c = J.jenga_test_gemm(a, b, out_f32=True, bn=bn)
    J.jenga_check_device_status()
    ref = a.float() @ b.float().t()
    err = (c - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-4, err
    if bn == 256:
        cb = J.jenga_test_gemm(a, b, out_f32=False, bn=bn)
        assert (cb.float() - ref).abs().max().item() / ref.abs().max().item() < 1e-2


# ------------------------------------------------------------------ scoring
def test_score_fp32_workload_against_oracle(J):
    c = synth.gen_score_case(0)
    q = torch.from_numpy(c.q).cuda()
    k = torch.from_numpy(c.k).cuda()
    sc = J.jenga_score_blocks(q, k, c.H, c.D, c.blk)
    J.jenga_check_device_status()
    ref = osc.block_scores_softmax_mass(c.q.reshape(c.S, c.H, c.D).astype(np.float64),
                                        c.k.reshape(c.S, c.H, c.D).astype(np.float64), c.blk)
    got = sc.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() / np.abs(ref).max() < 1e-3
    assert np.all(np.abs(got - ref) / ref < 1e-3)
    assert abs(got.sum() - c.H * c.S) < 1e-3 * c.H * c.S
    # selection: GPU scores through the oracle's mean threshold -> bit-exact indices
    idx, nk, mask = J.jenga_select(sc, "mean_ge")
    (oi, on, om), mean = osel.select_mean_ge(sc.cpu().numpy())
    assert int(nk[0]) == on and (idx.cpu().numpy() == oi).all() and (mask.cpu().numpy() == om).all()
    # gathered [n_kept * 32, 256] X and the scatter-add of 2 x the gathered rows
    x = torch.from_numpy(c.x).cuda()
    n_rows = on * c.blk
    xg = J.jenga_gather(x, idx, nk, c.blk, n_rows)
    ref_g = omv.gather(c.x.astype(np.float64), oi, on, c.blk)
    assert np.array_equal(xg.cpu().numpy().astype(np.float64), ref_g)
    x2 = x.clone()
    J.jenga_scatter_add(x2, xg, idx, nk, c.blk, 2.0)
    ref_s = omv.scatter_add(c.x.astype(np.float64), ref_g, oi, on, c.blk, 2.0, "f32")
    assert np.array_equal(x2.cpu().numpy().astype(np.float64), ref_s)
    J.jenga_check_device_status()


@pytest.mark.parametrize("S,H,causal", [(512, 2, True), (1024, 3, True), (256, 2, False)])
def test_score_bf16_against_oracle(J, S, H, causal):
    g = torch.Generator(device="cuda").manual_seed(S + H)
    q = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.25).to(torch.bfloat16)
    k = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.25).to(torch.bfloat16)
    sc = J.jenga_score_blocks(q, k, H, 128, 64, causal=causal)
    J.jenga_check_device_status()
    ref = osc.block_scores_softmax_mass(torch_to_f64(q).reshape(S, H, 128), torch_to_f64(k).reshape(S, H, 128), 64,
                                        causal=causal)
    got = sc.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) / np.abs(ref) < 2e-2), np.abs(got - ref).max()
    assert abs(got.sum() - H * S) < 2e-3 * H * S


@pytest.mark.parametrize("B,S,H,blk,causal", [(1, 4160, 2, 64, True), (1, 4160, 2, 64, False), (1, 1024, 3, 32, True),
                                             (1, 1056, 2, 32, False), (1, 2048, 4, 128, True), (1, 96, 2, 32, True),
                                             (3, 320, 2, 64, True), (2, 640, 1, 128, False)])
def test_score_bf16_shapes_against_oracle(J, B, S, H, blk, causal):
    """Single-pass scoring at ragged lengths (S % 128 = 64 or 32: a partial last query and
    key tile), 32-key chunks (blk 32), blk 128, S below one tile, and several sequences (the
    tile rows past a sequence's end belong to the next one and must be masked)."""
    g = torch.Generator(device="cuda").manual_seed(S * 7 + H + blk)
    q = (torch.randn(B, S, H * 128, device="cuda", generator=g) * 0.3).to(torch.bfloat16)
    k = (torch.randn(B, S, H * 128, device="cuda", generator=g) * 0.3).to(torch.bfloat16)
    sc = J.jenga_score_blocks(q, k, H, 128, blk, causal=causal)
    J.jenga_check_device_status()
    got = sc.cpu().numpy().astype(np.float64)
    for b in range(B):
        ref = osc.block_scores_softmax_mass(torch_to_f64(q[b]).reshape(S, H, 128), torch_to_f64(k[b]).reshape(S, H, 128),
                                            blk, causal=causal)
        assert np.all(np.abs(got[b] - ref) / np.abs(ref) < 2e-2), (b, np.abs(got[b] - ref).max())
        assert abs(got[b].sum() - H * S) < 2e-3 * H * S


def test_score_bf16_32_heads_s4096_and_row_lse(J):
    """The layer workload's scoring shape (32 heads x 128, S 4096, blocks of 64) against the
    oracle, and the row log-sum-exps the kernel leaves at the start of its workspace against
    the oracle's for a sample of rows."""
    S, H, blk = 4096, 32, 64
    g = torch.Generator(device="cuda").manual_seed(4096)
    q = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.2).to(torch.bfloat16)
    k = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.2).to(torch.bfloat16)
    lib = J._lib.load()
    ws = torch.zeros(lib.jenga_score_workspace_bytes(1, S, H, 128, blk), dtype=torch.uint8, device="cuda")
    sc = J.jenga_score_blocks(q, k, H, 128, blk, ws=ws)
    J.jenga_check_device_status()
    qf = torch_to_f64(q).reshape(S, H, 128)
    kf = torch_to_f64(k).reshape(S, H, 128)
    from tests.oracle_pool import oracle_pool
    with oracle_pool() as pm:
        ref = osc.block_scores_softmax_mass(qf, kf, blk, pmap=pm)
    got = sc.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) / np.abs(ref) < 2e-2), np.abs(got - ref).max()
    off = (-ws.data_ptr()) % 256
    neg_l2 = ws[off:off + H * S * 4].view(torch.float32).reshape(H, S).double().cpu().numpy()
    rows = np.r_[0, 1, 127, 128, 129, 2047, 4095, np.random.default_rng(0).integers(0, S, 24)]
    for h in (0, 17, 31):
        want = osc.row_lse(qf[:, h], kf[:, h], rows) / np.log(2.0)  # log2 units
        got_l = -neg_l2[h, rows]
        err = np.abs(got_l - want)
        assert np.all(err <= 2e-4 * (1 + np.abs(want))), (h, [(int(r), float(a), float(b)) for r, a, b in
                                                             zip(rows[:8], got_l[:8], want[:8])], float(err.max()))


def test_score_bf16_large_logit_jump(J):
    # one key far along the sequence whose logit exceeds every earlier one by > 60 (log2
    # units): rows that reach it must leave the pass-1 fast path and rescale exactly
    S, H, D = 1024, 2, 128
    g = torch.Generator(device="cuda").manual_seed(21)
    u = torch.randn(H * D, device="cuda", generator=g)
    q = (u + 0.5 * torch.randn(S, H * D, device="cuda", generator=g)).to(torch.bfloat16)
    k = (0.25 * torch.randn(S, H * D, device="cuda", generator=g))
    k[700] = 8.0 * u
    k = k.to(torch.bfloat16)
    sc = J.jenga_score_blocks(q, k, H, D, 64)
    J.jenga_check_device_status()
    ref = osc.block_scores_softmax_mass(torch_to_f64(q).reshape(S, H, D), torch_to_f64(k).reshape(S, H, D), 64)
    got = sc.cpu().numpy().astype(np.float64)
    assert ref[700 // 64] > 0.5 * H * (S - 700)  # the salient key's block takes most of the mass
    # blocks past the salient key score ~1e-33: their pairs sit below the fp32 normal range
    # (2^-126), where ex2 flushes and the FMA-pipe exponential floors at 2^-125, so the
    # relative bar gets an absolute allowance of 2^-124 per (query, key, head) pair
    floor = H * S * 64 * 2.0 ** -124
    assert np.all(np.abs(got - ref) <= 2e-2 * np.abs(ref) + floor), np.abs(got - ref).max()
    big = ref > 1e-20
    assert np.all(np.abs(got - ref)[big] / ref[big] < 2e-2)
    assert abs(got.sum() - H * S) < 2e-3 * H * S


def test_exp2_fma_against_float64(J):
    # the FMA-pipe exponential (cubic after a binary split) that scoring uses for part of
    # its columns: relative error of the fitted cubic is 7.5e-5; clamped outside [-125, 64]
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.cat([torch.linspace(-125.0, 64.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 20, device="cuda", generator=g) * 40.0 - 30.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, -124.75, 63.5], device="cuda")])
    y_fma, y_mufu = J._api_test_exp2(x)
    xd = x.double().cpu()
    ref = torch.exp2(xd)
    rel = ((y_fma.double().cpu() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    rel_mufu = ((y_fma.double() - y_mufu.double()).abs() / y_mufu.double()).max().item()
    assert rel_mufu < 2e-4, rel_mufu
    lo = J._api_test_exp2(torch.tensor([-200.0, -1e30, -float("inf")], device="cuda"))[0].double().cpu()
    assert torch.all(lo <= 2.0 ** -125 * 1.5) and torch.all(lo > 0)
    hi = J._api_test_exp2(torch.tensor([100.0, 1e30], device="cuda"))[0].double().cpu()
    assert torch.all(torch.isfinite(hi)) and torch.all(hi >= 2.0 ** 63)


def test_score_bf16_fused_qk_buffer_and_batch(J):
    S, H = 512, 2
    g = torch.Generator(device="cuda").manual_seed(7)
    qk = (torch.randn(2, S, 2 * H * 128, device="cuda", generator=g) * 0.3).to(torch.bfloat16)
    sc = J.jenga_score_blocks(qk[:, :, :H * 128], qk[:, :, H * 128:], H, 128, 128)
    for b in range(2):
        qb = torch_to_f64(qk[b, :, :H * 128]).reshape(S, H, 128)
        kb = torch_to_f64(qk[b, :, H * 128:]).reshape(S, H, 128)
        ref = osc.block_scores_softmax_mass(qb, kb, 128)
        assert np.all(np.abs(sc[b].cpu().numpy() - ref) / ref < 2e-2)


def test_score_paper_blockmax(J):
    S, H, D, blk = 64, 2, 16, 8
    g = torch.Generator(device="cuda").manual_seed(9)
    q = torch.randn(S, H * D, device="cuda", generator=g, dtype=torch.float32)
    k = torch.randn(S, H * D, device="cuda", generator=g, dtype=torch.float32)
    sc = J.jenga_score_blocks(q, k, H, D, blk, mode="paper_blockmax")
    ref = osc.block_scores_paper_blockmax(torch_to_f64(q).reshape(S, H, D), torch_to_f64(k).reshape(S, H, D), blk)
    assert np.allclose(sc.cpu().numpy(), ref, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("S,H,blk,causal", [(4096, 32, 64, True), (1024, 3, 32, True), (1024, 2, 128, False),
                                             (2048, 2, 256, True), (4160, 2, 64, True), (640, 4, 128, True)])
def test_score_paper_blockmax_bf16_tcgen05(J, S, H, blk, causal):
    """Eq. (2) block-max scores on the tensor-core path (bf16, head_dim 128) against the
    oracle's block_scores_paper_blockmax on the same bf16 values: blocks of 32, 64, 128
    and 256 tokens (several 128-token sub-tiles per block), a ragged S, causal and not."""
    g = torch.Generator(device="cuda").manual_seed(S + H + blk)
    q = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.5).to(torch.bfloat16)
    k = (torch.randn(S, H * 128, device="cuda", generator=g) * 0.5).to(torch.bfloat16)
    sc = J.jenga_score_blocks(q, k, H, 128, blk, causal=causal, mode="paper_blockmax")
    J.jenga_check_device_status()
    ref = osc.block_scores_paper_blockmax(torch_to_f64(q).reshape(S, H, 128), torch_to_f64(k).reshape(S, H, 128), blk,
                                          causal=causal)
    got = sc.cpu().numpy().astype(np.float64)
    rel = np.abs(got - ref) / np.abs(ref)
    assert np.all(rel < 2e-3), rel.max()


# ------------------------------------------------------------------ selection
@pytest.mark.parametrize("nb,mode,param,dist", [(256, "topk_frac", 0.8, "normal"), (256, "topk_frac", 0.4, "ties"),
                                               (16, "mean_ge", 0, "normal"), (1000, "mean_ge", 0, "ties"),
                                               (8192, "abs_ge", 0.5, "normal"), (300, "topk", 7, "ties"),
                                               (64, "topk_frac", 0.0, "normal"), (64, "topk_frac", 1.0, "normal")])
def test_select_bit_exact(J, nb, mode, param, dist):
    sc = synth.gen_scores(nb, 3, nb, dist)
    idx, nk, mask = J.jenga_select(torch.from_numpy(sc).cuda(), mode, param)
    J.jenga_check_device_status()
    oi, on, om = osel.select(sc, mode, param)
    assert np.array_equal(nk.cpu().numpy(), on)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.array_equal(mask.cpu().numpy(), om)


@pytest.mark.parametrize("mode,param,nb", [("abs_ge", 0.25, (1 << 20) + 777), ("mean_ge", 0, (1 << 20) + 777),
                                           ("abs_ge", 0.5, 1 << 22), ("mean_ge", 0, (1 << 22) + 4)])
def test_select_large_multi_cta(J, mode, param, nb):
    # single-pass look-back compaction: ragged tails (scalar loads) and multiples of 4
    # (vector loads, 16-byte mask stores)
    sc = synth.gen_scores(5, 2, nb)
    idx, nk, mask = J.jenga_select(torch.from_numpy(sc).cuda(), mode, param)
    J.jenga_check_device_status()
    for b in range(2):
        if mode == "abs_ge":
            oi, on, om = osel.select_abs_ge(sc[b], param)
        else:
            (oi, on, om), _ = osel.select_mean_ge(sc[b])
        assert int(nk[b]) == on
        assert np.array_equal(idx[b].cpu().numpy(), oi)
        assert np.array_equal(mask[b].cpu().numpy(), om)


# ------------------------------------------------------------------ movement
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gather_scatter_random(J, dtype):
    S, h, blk = 1024, 384, 64
    g = torch.Generator(device="cuda").manual_seed(11)
    x = torch.randn(S, h, device="cuda", generator=g).to(dtype)
    sc = synth.gen_scores(12, 1, S // blk)
    idx, nk, _ = J.jenga_select(torch.from_numpy(sc).cuda(), "topk_frac", 0.5)
    n_cap = (S // blk) * blk
    out = torch.full((n_cap, h), 7.0, device="cuda", dtype=dtype)
    J.jenga_gather(x, idx, nk, blk, n_cap, out=out)
    xi = idx.cpu().numpy()[0]
    n = int(nk[0])
    ref = omv.gather(torch_to_f64(x), xi, n, blk)
    assert np.array_equal(torch_to_f64(out[: n * blk]), ref)
    assert (out[n * blk:] == 7.0).all()
    y = torch.randn(n * blk, h, device="cuda", generator=g).to(dtype)
    x2 = x.clone()
    J.jenga_scatter_add(x2, y, idx, nk, blk, 1.0)
    ref2 = omv.scatter_add(torch_to_f64(x), torch_to_f64(y), xi, n, blk, 1.0,
                           "bf16" if dtype == torch.bfloat16 else "f32")
    assert np.array_equal(torch_to_f64(x2), ref2)
    # keep-none: nothing moves
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    x3 = x.clone()
    J.jenga_scatter_add(x3, y, idx, z, blk, 1.0)
    assert torch.equal(x3, x)


def test_gather_scatter_batched_pitched(J):
    # two sequences, rows 136 bf16 wide (17 vectors: an odd divisor for the row split) inside
    # a 200-wide pitch, block 32 (544 vectors per block: one partial chunk per block)
    B, S, h, W, blk = 2, 2048, 136, 200, 32
    g = torch.Generator(device="cuda").manual_seed(13)
    xw = torch.randn(B, S, W, device="cuda", generator=g).to(torch.bfloat16)
    x = xw[:, :, :h]
    sc = synth.gen_scores(14, B, S // blk)
    idx, nk, _ = J.jenga_select(torch.from_numpy(sc).cuda(), "topk_frac", 0.3)
    n_cap = (S // blk) * blk
    out = J.jenga_gather(x, idx, nk, blk, n_cap)
    yw = torch.randn(B, n_cap, W, device="cuda", generator=g).to(torch.bfloat16)
    y = yw[:, :, :h]
    xw2 = xw.clone()
    J.jenga_scatter_add(xw2[:, :, :h], y, idx, nk, blk, 0.5)
    for b in range(B):
        xi = idx.cpu().numpy()[b]
        n = int(nk[b])
        assert np.array_equal(torch_to_f64(out[b, : n * blk]), omv.gather(torch_to_f64(x[b]), xi, n, blk))
        ref = omv.scatter_add(torch_to_f64(x[b]), torch_to_f64(y[b, : n * blk]), xi, n, blk, 0.5, "bf16")
        assert np.array_equal(torch_to_f64(xw2[b, :, :h]), ref)
    assert torch.equal(xw2[:, :, h:], xw[:, :, h:]), "the pitch padding is never written"
    J.jenga_check_device_status()


def test_scale_rows(J):
    x = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    rows = torch.tensor([3, 17, 40], dtype=torch.int32, device="cuda")
    y = x.clone()
    J.jenga_scale_rows(y, rows, 3.0)
    ref = torch_to_f64(x)
    ref[[3, 17, 40]] = torch_to_f64(x[[3, 17, 40]].float().mul(3).to(torch.bfloat16))
    assert np.array_equal(torch_to_f64(y), ref)


# ------------------------------------------------------------------ predictor
def test_predictor_against_oracle(J):
    shape = synth.LayerShape(hidden=512, heads=4, head_dim=128, ffn=1024)
    case = synth.gen_layer_case(4, S=2048, blk=128, shape=shape, salient_frac=0.0, predictor_hidden=128)
    pr = case.predictor
    x = bits_to_torch(case.x)
    w1 = bits_to_torch(pr["w1"])
    w2 = bits_to_torch(pr["w2"]).reshape(-1)
    b1 = torch.from_numpy(pr["b1"]).cuda()
    b2 = torch.from_numpy(pr["b2"]).cuda()
    s = J.jenga_predict_blocks(x, 128, w1, b1, w2, b2)
    J.jenga_check_device_status()
    ref = opr.predict_blocks(from_bits(case.x), 128, from_bits(pr["w1"]), pr["b1"], from_bits(pr["w2"]), pr["b2"])
    got = s.cpu().numpy().astype(np.float64)
    assert rel_max(got, ref) < 1e-3


# ------------------------------------------------------------------ Q/K predictor pair (Eq. 3)
@pytest.mark.parametrize("S,h,blk,r1,r2,d,causal,B", [(2048, 512, 128, 128, 64, 16, True, 1),
                                                      (1024, 264, 64, 40, 24, 1, True, 2),
                                                      (4096, 5120, 128, 128, 128, 32, False, 1)])
def test_predictor_pair_against_oracle(J, S, h, blk, r1, r2, d, causal, B):
    g = torch.Generator(device="cpu").manual_seed(S + d)
    x = torch.randn(B, S, h, generator=g).to(torch.bfloat16)
    mk = lambda: tuple((torch.randn(*shp, generator=g) * sd).to(torch.bfloat16)
                       for shp, sd in (((r1, h), 0.02), ((r2, r1), 0.1), ((d, r2), 0.1)))
    qw, kw = mk(), mk()
    got = J.jenga_predict_blocks_qk(x.cuda(), blk, tuple(t.cuda() for t in qw), tuple(t.cuda() for t in kw),
                                    causal=causal)
    J.jenga_check_device_status()
    f64 = lambda t: t.to(torch.float64).numpy()
    for b in range(B):
        ref = opr.predict_blocks_qk(f64(x[b]), blk, tuple(f64(t) for t in qw), tuple(f64(t) for t in kw), causal)
        assert rel_max(got[b].cpu().numpy().astype(np.float64), ref) < 1e-3


# ------------------------------------------------------------------ MLP-block criterion (§4.2.4)
@pytest.mark.parametrize("n_cap,n_kept,blk,F,pitch", [(64, 50, 64, 11008, 11008), (33, 33, 32, 520, 528),
                                                      (16, 0, 128, 256, 256)])
def test_mlp_block_scores_and_second_list(J, n_cap, n_kept, blk, F, pitch):
    from oracle import mlp_blocks as omb
    g = torch.Generator(device="cpu").manual_seed(n_cap + F)
    aw = (torch.randn(n_cap * blk, pitch, generator=g) * torch.rand(n_cap * blk, 1, generator=g) * 3).to(torch.bfloat16)
    a = aw.cuda()[:, :F]
    nk = torch.tensor([n_kept], dtype=torch.int32, device="cuda")
    sc = J.jenga_mlp_block_scores(a, blk, nk)
    J.jenga_check_device_status()
    ref = omb.mlp_block_scores(aw[:, :F].to(torch.float64).numpy(), blk, n_kept)
    got = sc.cpu().numpy().astype(np.float64)
    assert np.all(np.isneginf(got[n_kept:]))
    if n_kept:
        assert np.all(np.abs(got[:n_kept] - ref[:n_kept]) / ref[:n_kept] < 1e-5)
    # second index list: the MLP keeps half of the attention-retained blocks (GPU scores
    # through the oracle's selection, bit-exact), composed with an attention list
    k = (n_kept + 1) // 2
    pos, npos, _ = J.jenga_select(sc[None], "topk", float(k))
    opos, onpos, _ = osel.select_topk(got, k)
    assert int(npos[0]) == onpos and np.array_equal(pos.cpu().numpy()[0], opos)
    outer = torch.arange(0, 2 * n_cap, 2, dtype=torch.int32, device="cuda")  # attention list: even blocks
    inner = J.jenga_compose_block_indices(outer, pos[0], npos)
    want = omb.compose_indices(outer.cpu().numpy(), opos, onpos)
    assert np.array_equal(inner.cpu().numpy(), want)
