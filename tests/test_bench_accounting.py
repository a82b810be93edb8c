"""The bench's work accounting against figures derived independently from the model shapes."""
import bench
import krea2_inputs as KI


def test_gemm_flops_per_token():
    # 2 * (6144 * 15360 + 6144 * 6144 + 6144 * 32768 + 16384 * 6144) = 868.2 MFLOP per token
    d = KI.FULL
    per_token = 2 * (d.C * d.qkvg_cols + d.HD * d.C + d.C * 2 * d.F + d.F * d.C)
    assert per_token == 868_220_928
    w = bench.block_kernel_work(d, 1, 0, 1, [])
    gemm = sum(w[k]["flops"] for k in ("qkv_proj", "out_proj_resid", "gate_up_swiglu", "down_proj_resid"))
    assert gemm == per_token


def test_block_1024sq_cfg_flops():
    # 9216 tokens of GEMM work + attention over 4608 queries x (512 + 4096) and x (8 + 4096) valid keys
    wl = KI.block_1024_cfg()
    d = wl.dims
    fl = bench.block_flops(d, wl.B, wl.T, wl.N, wl.lengths)
    gemm = 868_220_928 * 9216
    attn = 4 * 128 * 48 * 4608 * ((512 + 4096) + (8 + 4096))
    assert fl == gemm + attn
    assert abs(fl / 1e12 - 8.99) < 0.01


def test_backbone_step_flops():
    wl = KI.backbone_1024()
    fl = bench.backbone_flops(wl.dims, wl.B, wl.T, wl.N, wl.lengths)
    assert abs(fl / 1e12 - 126.64) < 0.01     # 28 x 4.523 TFLOP + time path, img_in, final layer


def test_norm_bytes():
    d = KI.FULL
    w = bench.block_kernel_work(d, 1, 512, 4096, [512])
    assert w["norm1"]["bytes"] == 4608 * 6144 * 6      # fp32 in, bf16 out


def test_kv_cache_step_flops():
    # 4096 target queries over 512 valid text + 4096 cached condition-image + 4096 own keys
    d = KI.FULL
    fl = bench.kv_step_flops(d, 4096, 512 + 4096 + 4096)
    assert fl == 4 * 128 * 48 * 4096 * 8704
    assert abs(fl / 1e12 - 0.8762) < 1e-3


def test_both_arms_print_the_same_config():
    wl = KI.backbone_1024()
    c = bench.workload_config(wl, 1)
    assert c["workload"] == wl.name and c["seq_len"] == 4608 and c["layers"] == 28
    assert abs(c["flops_per_step"] / 1e12 - 126.64) < 0.01
    assert c["parallelism"] == "single GPU" and bench.workload_config(wl, 8)["parallelism"] == "replicas"


def test_rank_layout_guards_the_rank_count():
    import pytest
    assert bench.rank_layout(1, {}) == (0, 1, 0)
    assert bench.rank_layout(4, {}) == "spawn"                      # no launcher: bench starts the ranks
    env = {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}
    assert bench.rank_layout(2, env) == (1, 2, 1)
    with pytest.raises(SystemExit):
        bench.rank_layout(8, env)                                    # launcher and --gpus disagree
    with pytest.raises(SystemExit):
        bench.rank_layout(0, {})


def test_summary_fits_the_tail_of_the_line():
    # the driver keeps the last 1500 characters of the bench's output: the summary must fit in them
    import json
    pk = {"bf16_tflops": 1683.8, "bf16_tflops_sustained": 1391.3, "hbm_gbs": 6540.2, "source": "measured"}
    names = ("modulation", "norm1", "qkv_proj", "attention", "out_proj_resid", "norm2", "gate_up_swiglu",
             "down_proj_resid")
    kern = {k: ({"ms": 0.123456, "tflops": 1234.5678, "frac_sustained": 0.87654, "share": 0.1}
                if "proj" in k or k in ("attention", "gate_up_swiglu") else
                {"ms": 0.0456789, "gbs": 4567.891, "frac_hbm": 0.698765, "share": 0.01}) for k in names}
    cfg = {"ms_per_block": 7.2012345, "tflops": 1248.98765, "frac_burst": 0.7421234, "frac_sustained": 0.898765,
           "kernels": kern}
    sweep = [{"grid": g, "ms": 0.1234567, "tflops": 987.654321} for g in (32, 64, 96, 128)]
    s = json.dumps({"summary": bench.summary(1119.123456, 113.123456, pk, cfg, kern, sweep)})
    assert len(s) < 1300, len(s)
