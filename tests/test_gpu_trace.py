"""Tracing (gptq_trace_enable / gptq_trace_read): every kernel the library
launches while tracing is on is accounted for, under its own name, with a
positive device time; a read empties the record."""
import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq
    import synth_inputs as si


def test_trace_accounts_for_every_launch_of_a_layer_pass():
    spec = si.scaled(si.SPECS["attn4096"], rows=256, n=512, n_tok=4096)
    W, X = si.make_layer(spec, "cuda")
    torch.cuda.synchronize()
    gq.gptq_trace_read()  # drop anything recorded earlier
    gq.gptq_trace_enable(True)
    try:
        n0 = gq.gptq_kernel_launches()
        gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block)
        n1 = gq.gptq_kernel_launches()
        tr = gq.gptq_trace_read()
    finally:
        gq.gptq_trace_enable(False)
    assert sum(launches for launches, _ in tr.values()) == n1 - n0
    for name in ("syrk_tc_kernel", "chol_tc_kernel", "gptq_block_kernel<16>", "trailing_tc_kernel", "pack_kernel<4>"):
        assert name in tr, sorted(tr)
        assert tr[name][0] >= 1 and tr[name][1] > 0.0
    assert tr["gptq_block_kernel<16>"][0] == 4  # 512 columns in blocks of 128
    assert gq.gptq_trace_read() == {}
    # tracing off: launches are not recorded
    gq.gptq_pack(torch.zeros((4, 64), dtype=torch.uint8, device="cuda"), 4)
    torch.cuda.synchronize()
    assert gq.gptq_trace_read() == {}
