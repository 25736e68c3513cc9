"""Helpers shared by the GPU parity tests (conversions only)."""
import numpy as np
import torch


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cache_arrays(cache, NB: int) -> dict:
    """The cache's arrays restricted to the slots the oracle builds."""
    NU = -(-cache.n_tokens // 4)
    return dict(
        U=cache.U[:, :NU].cpu().numpy(),
        bucket_of_unit=cache.bucket_of_unit[:, :NU].cpu().numpy(),
        members=cache.members[:, :NU].cpu().numpy(),
        offsets=cache.offsets[:, :NB + 1].cpu().numpy(),
        cnt_lr=cache.cnt_lr[:, :NB].cpu().numpy(),
        minlr=cache.minlr[:, :NB].cpu().numpy(),
        maxpos=cache.maxpos[:, :NB].cpu().numpy(),
        sum=cache.sum[:, :NB].cpu().numpy(),
        cent=bits(cache.cent[:, :NB]),
    )


def oracle_cfg(cfg):
    import oracle
    return oracle.Cfg(k=cfg.k, sinks=cfg.sinks, window=cfg.window, beam=cfg.beam, mode=cfg.mode,
                      agg=cfg.agg)
