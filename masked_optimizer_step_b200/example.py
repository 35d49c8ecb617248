"""Usage example: one sparse step on one 4096 x 4096 projection through the Python binding.

    python -m masked_optimizer_step_b200.example

Masks from the row tracker (the forward outputs Y), the masked weight gradient of the active
rows on the tensor cores, then the fused update. Needs a B200 and the built library.
"""
import torch

from masked_optimizer_step_b200 import binding as sf


def main():
    R, C, T = 4096, 4096, 2048
    mat = sf.Matrix(R, C, slot_cap=128)                # int8 + scale + residual, live bf16, moments
    sf.sf_mask_init(mat.mask)
    sf.sf_quantize_init(torch.randn(R, C, device="cuda") * 0.02, mat)

    gain = torch.full((R,), 1e-3, device="cuda")
    gain[torch.randperm(R, device="cuda")[:41]] = 1.0            # ~1% of rows carry the signal
    Y = (torch.randn(T, R, device="cuda") * gain).to(torch.bfloat16)  # forward outputs (row tracker)
    dX = torch.randn(T, R, device="cuda", dtype=torch.bfloat16)  # output gradients
    A = torch.randn(T, C, device="cuda", dtype=torch.bfloat16)   # layer inputs
    status = sf.status_word()

    sf.sf_mask_update([mat.mask], [sf.make_src(sf.SF_SRC_OUTPUT_BF16, Y, n=T, ld=Y.stride(0))], 0.01, status)
    probs = [sf.dw_problem(dX, A, mat.mask, mat.grad)]
    sf.sf_masked_dw(probs, status, ws=sf.dw_workspace(probs))
    sf.sf_sparse_update([sf.matrix_struct(mat)], sf.AdamParams(), status)
    assert int(status[0]) == 0      # SF_STATUS_* bits: slot overflow, non-finite, bad token, timeout
    return int(mat.mask.counts[0])  # active rows this step


if __name__ == "__main__":
    print(f"active rows: {main()}")
