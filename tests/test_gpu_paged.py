"""Paged KV cache: append with online scale update, and decode over pages.

qk4v8_kv_append writes new tokens into 128-token pages. K rows are quantized on
their own; every V group of 32 tokens that new tokens touch gets its scale
recomputed over all of its tokens (the open group's earlier tokens come from
the bf16 staging buffer), so after any sequence of appends the pages must hold
exactly the bytes that quantizing the whole sequence at once gives: the oracle
is oracle.quantize_qk / quantize_v over the concatenated sequence. The paged
decode calls must equal the contiguous ones bit for bit (same tiles, same
arithmetic) and match the fp64 oracle within the attention tolerance.
"""
import numpy as np
import pytest
import torch

import bit_quantized_attention_qk4v8_b200 as qk
import oracle
import synth
from gpu_util import assert_close, to_dev
from layouts import gather_pages, qk_scales_logical, unpack_e2m1, v_scales_logical

pytestmark = pytest.mark.gpu


def _inputs(B, T, Hkv, seed, k_out=2):
    wl = synth.Workload("p", "decode", B=B, Hq=Hkv, Hkv=Hkv, Sq=1, Lk=T, seed=seed, k_outliers=k_out,
                        outlier_mult=16.0)
    return wl.generate()


def _block_table(B, max_pages, num_pages, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)[:B * max_pages]
    return torch.from_numpy(perm.reshape(B, max_pages).astype(np.int32))


def _check_cache(cache, kbits, vbits, L, hadamard_k=False):
    """Pages hold the oracle's quantization of tokens [0, L) (every sequence L long)."""
    nb = (L + 127) // 128
    bt = cache.block_table.cpu().numpy()
    kc, ks = gather_pages(cache.k_codes.cpu().numpy(), cache.k_scales.cpu().numpy(), bt, nb)
    vc, vs = gather_pages(cache.v_codes.cpu().numpy(), cache.v_scales.cpu().numpy(), bt, nb)
    B = kbits.shape[0]
    if hadamard_k:
        ok_c, ok_s = oracle.quantize_qk_hadamard(kbits[:, :L])
    else:
        ok_c, ok_s = oracle.quantize_qk(kbits[:, :L])
    ov_c, ov_s = oracle.quantize_v(vbits[:, :L], np.full((B,), L, np.int32))
    assert np.array_equal(unpack_e2m1(kc[:, :, :L]), ok_c), f"K codes at length {L}"
    assert np.array_equal(qk_scales_logical(ks, L), ok_s), f"K scales at length {L}"
    assert np.array_equal(vc[..., :L], ov_c), f"V codes at length {L}"
    assert np.array_equal(v_scales_logical(vs, L), ov_s), f"V scales at length {L}"
    # The open V group's codes past L are written as zero.
    if L % 32:
        assert not vc[..., L:(L + 31) // 32 * 32].any()


@pytest.mark.parametrize("hadamard_k", [False, True])
def test_append_sequence_matches_whole_sequence_quantization(hadamard_k):
    B, Hkv, T = 3, 2, 300
    chunks = [37, 1, 1, 8, 95, 1, 8, 31, 1, 64, 3, 50]
    assert sum(chunks) == T
    gen = _inputs(B, T, Hkv, seed=21)
    k, v = to_dev(gen["k"]), to_dev(gen["v"])
    max_pages, num_pages = 3, 16
    cache = qk.paged_kv(B, Hkv, num_pages, _block_table(B, max_pages, num_pages, 3), hadamard_k=hadamard_k)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    L = 0
    for n in chunks:
        qk.kv_append(cache, k[:, L:L + n], v[:, L:L + n], dev_status=status)   # strided views
        L += n
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert cache.seqlens.cpu().tolist() == [L] * B
        _check_cache(cache, gen["k"], gen["v"], L, hadamard_k)


def test_append_whole_prompt_then_tokens():
    B, Hkv, T = 2, 8, 1100
    gen = _inputs(B, T, Hkv, seed=22, k_out=4)
    k, v = to_dev(gen["k"]), to_dev(gen["v"])
    cache = qk.paged_kv(B, Hkv, 40, _block_table(B, 9, 40, 4))
    qk.kv_append(cache, k[:, :1000].contiguous(), v[:, :1000].contiguous())
    for L in range(1000, T, 25):
        qk.kv_append(cache, k[:, L:L + 25], v[:, L:L + 25])
    torch.cuda.synchronize()
    _check_cache(cache, gen["k"], gen["v"], T)


def test_append_with_separate_length_output():
    """seqlens_out distinct from seqlens: the append kernel writes the new lengths
    itself and leaves the input lengths as they were."""
    from bit_quantized_attention_qk4v8_b200._lib import lib
    B, Hkv, T = 3, 4, 70
    gen = _inputs(B, T, Hkv, seed=23)
    k, v = to_dev(gen["k"]), to_dev(gen["v"])
    cache = qk.paged_kv(B, Hkv, 8, _block_table(B, 2, 8, 5))
    qk.kv_append(cache, k[:, :45].contiguous(), v[:, :45].contiguous())
    lens_out = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    kn, vn = k[:, 45:].contiguous(), v[:, 45:].contiguous()
    st = lib().qk4v8_kv_append(kn.data_ptr(), vn.data_ptr(), B, T - 45, Hkv, 128, kn.stride(0), kn.stride(1),
                               kn.stride(2), cache.seqlens.data_ptr(), lens_out.data_ptr(),
                               cache.block_table.data_ptr(), cache.max_pages, cache.num_pages,
                               cache.k_codes.data_ptr(), cache.k_scales.data_ptr(), cache.v_codes.data_ptr(),
                               cache.v_scales.data_ptr(), cache.v_tail.data_ptr(), 0, None,
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert cache.seqlens.cpu().tolist() == [45] * B
    assert lens_out.cpu().tolist() == [T] * B
    cache.seqlens.copy_(lens_out)
    _check_cache(cache, gen["k"], gen["v"], T)


def _paged_from_contiguous(kp, vp, max_pages, num_pages, seed):
    """A page pool holding the contiguous cache's blocks in a random page order."""
    B, H = kp.B, kp.H
    bt = _block_table(B, max_pages, num_pages, seed)
    cache = qk.paged_kv(B, H, num_pages, bt)
    idx = bt.long().cuda()
    for i in range(max_pages):
        pages = idx[:, i]
        cache.k_codes[pages] = kp.codes[:, :, i * 128:(i + 1) * 128]
        cache.k_scales[pages] = kp.scales[:, :, i]
        cache.v_codes[pages] = vp.codes[:, :, i]
        cache.v_scales[pages] = vp.scales[:, :, i]
    return cache


@pytest.mark.parametrize("Hq,Hkv,nq,causal,window,splits", [
    (32, 8, 1, True, 0, 0),       # swap-AB kernel, one split
    (16, 4, 8, True, 0, 3),       # swap-AB kernel, splits and merge
    (64, 8, 8, True, 0, 2),       # GQA kernel, balanced schedule
    (64, 8, 8, False, 512, 0),    # GQA kernel, draft-block window
    (16, 2, 8, False, 300, 2),    # swap-AB kernel, window and splits
])
def test_paged_decode_equals_contiguous(Hq, Hkv, nq, causal, window, splits):
    lens = [1500, 700, 1281, 64]
    wl = synth.Workload("p", "decode", B=len(lens), Hq=Hq, Hkv=Hkv, Sq=nq, Lk=max(lens), seed=Hq + nq, k_outliers=4,
                        q_outliers=True, outlier_mult=16.0)
    gen = wl.generate()
    gen["seqlens"] = np.array(lens, np.int32)
    max_pages = 12
    sl = torch.from_numpy(gen["seqlens"]).cuda()
    kp = qk.quantize_qk(to_dev(gen["k"]), cap=max_pages * 128, seqlens=sl)
    vp = qk.quantize_v(to_dev(gen["v"]), cap=max_pages * 128, seqlens=sl)
    qp = qk.quantize_qk(to_dev(gen["q"]))
    cache = _paged_from_contiguous(kp, vp, max_pages, 64, seed=7)
    cache.seqlens.copy_(sl)
    ref = qk.attention_decode(qp, kp, vp, sl, max_seqlen=max(lens), causal_in_block=causal, num_splits=splits,
                              window=window)
    got = qk.attention_decode_paged(qp, cache, max_seqlen=max(lens), causal_in_block=causal, window=window,
                                    num_splits=splits)
    got16 = qk.attention_decode_bf16_paged(to_dev(gen["q"]), cache, max_seqlen=max(lens), causal_in_block=causal,
                                           window=window, num_splits=splits)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    oz = oracle.quantize_workload(gen)
    oref, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], gen["seqlens"],
                               causal=causal, window=window)
    assert_close(got16, oref, f"paged bf16 Hq={Hq} nq={nq} window={window}")


@pytest.mark.parametrize("Hq,Hkv,window", [(32, 8, 0), (64, 8, 1024)])
def test_decode_loop_over_appended_pages(Hq, Hkv, window):
    """Prompt appended to empty pages, then verify steps: append 8 tokens, attend
    (the 8 new tokens are the query block), against the oracle on the whole
    sequence at every step."""
    B, nq, prompt, steps = 2, 8, 1300, 4
    T = prompt + nq * steps
    wl = synth.Workload("p", "decode", B=B, Hq=Hq, Hkv=Hkv, Sq=nq * steps, Lk=T, seed=Hq, k_outliers=4,
                        outlier_mult=16.0)
    gen = wl.generate()
    k, v, qall = to_dev(gen["k"]), to_dev(gen["v"]), to_dev(gen["q"])
    cache = qk.paged_kv(B, Hkv, 64, _block_table(B, 12, 64, 9))
    qk.kv_append(cache, k[:, :prompt], v[:, :prompt])
    L = prompt
    for s in range(steps):
        qk.kv_append(cache, k[:, L:L + nq], v[:, L:L + nq])
        L += nq
        q = qall[:, s * nq:(s + 1) * nq]
        out = qk.attention_decode_bf16_paged(q, cache, max_seqlen=L, causal_in_block=window == 0, window=window)
        torch.cuda.synchronize()
        sub = dict(q=gen["q"][:, s * nq:(s + 1) * nq], k=gen["k"][:, :L], v=gen["v"][:, :L],
                   seqlens=np.full((B,), L, np.int32))
        oz = oracle.quantize_workload(sub)
        ref, _ = oracle.attention(oz["qc"], oz["qs"], oz["kc"], oz["ks"], oz["vc"], oz["vs"], sub["seqlens"],
                                  causal=window == 0, window=window)
        assert_close(out, ref, f"decode step {s} (L={L})")


def test_bad_page_entries_are_reported_not_followed():
    """Block-table entries outside the pool: the append skips those tokens and the
    attention reads page 0 instead; both report QK4V8_ERR_INVALID_ARG (1) in
    dev_status and leave the context usable."""
    B, Hkv = 2, 2
    gen = _inputs(B, 200, Hkv, seed=30)
    k, v = to_dev(gen["k"]), to_dev(gen["v"])
    bt = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32)     # page 99 does not exist (4 pages)
    cache = qk.paged_kv(B, Hkv, 4, bt)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    qk.kv_append(cache, k, v, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    status.zero_()
    qp = qk.quantize_qk(to_dev(_inputs(B, 1, 8, seed=31)["q"][:, :1]))
    qk.attention_decode_paged(qp, cache, max_seqlen=200, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    # The context still works.
    x = torch.ones(4, device="cuda")
    assert float(x.sum().item()) == 4.0
