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
