"""Device-resident quantised Mamba2 mixer layers and stacks.

PyTorch provides device memory and streams; every step (weight rotation and
quantisation, calibration, prefill, decode) runs in libfastmamba's kernels
through the ctypes binding in `lib`.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lib
from .synth import MixerShape


def _dev(a, dtype, device):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype).contiguous()


class DeviceLayer:
    """One prepared mixer layer: quantised weights + exponent table on the GPU."""

    def __init__(self, params: dict, shape: MixerShape, rotate: int = 1, mode: int = lib.FM_DYNAMIC,
                 prenorm: bool = False, device="cuda", stream=None):
        s = shape
        self.shape, self.rotate, self.mode, self.prenorm = s, rotate, mode, prenorm
        self.device = torch.device(device)
        f32 = lambda a: _dev(a, torch.float32, self.device)
        w_in, w_out = f32(params["w_in"]), f32(params["w_out"])
        self.w_in_q = torch.empty((s.n_in, s.d_model), dtype=torch.int8, device=self.device)
        self.w_in_s = torch.empty(s.n_in, dtype=torch.float32, device=self.device)
        self.w_out_q = torch.empty((s.d_model, s.d_inner), dtype=torch.int8, device=self.device)
        self.w_out_s = torch.empty(s.d_model, dtype=torch.float32, device=self.device)
        lib.prepare_linear(w_in, rotate, self.w_in_q, self.w_in_s, stream)
        lib.prepare_linear(w_out, rotate, self.w_out_q, self.w_out_s, stream)
        self.conv_w = f32(params["conv_w"])
        self.conv_b = f32(params["conv_b"])
        self.a_log = f32(params["a_log"])
        self.D = f32(params["D"])
        self.dt_bias = f32(params["dt_bias"])
        self.norm_w = f32(params["norm_w"])
        self.prenorm_w = f32(params["prenorm_w"]) if prenorm else None
        self.layout = lib.exp_table_layout(s)
        self.exps = torch.zeros(self.layout.size, dtype=torch.int32, device=self.device)
        self.conv_wq = torch.empty((s.conv_ch, 4), dtype=torch.int8, device=self.device)
        self.conv_bq = torch.zeros(s.conv_ch, dtype=torch.int32, device=self.device)
        self.A_q = torch.empty(s.nheads, dtype=torch.int32, device=self.device)
        self.D_q = torch.empty(s.nheads, dtype=torch.int32, device=self.device)
        self.static_amax = torch.zeros(4, dtype=torch.float32, device=self.device)
        lib.prepare_mixer_params(s, self.conv_w, self.a_log, self.D, self.conv_wq, self.A_q,
                                 self.D_q, self.exps, stream)
        del w_in, w_out
        self.struct = self._make_struct()
        p = lambda t: t.data_ptr()
        self.lq_struct = lib.fm_lq_params(p(self.conv_w), p(self.conv_b), p(self.a_log), p(self.D))

    def _make_struct(self) -> lib.fm_layer:
        p = lambda t: None if t is None else t.data_ptr()
        return lib.fm_layer(lib.shape_struct(self.shape), self.rotate, self.mode,
                            p(self.w_in_q), p(self.w_in_s), p(self.w_out_q), p(self.w_out_s),
                            p(self.prenorm_w), p(self.conv_wq), p(self.conv_bq), p(self.dt_bias),
                            p(self.A_q), p(self.D_q), p(self.norm_w), p(self.exps),
                            p(self.static_amax))

    # ------------------------------------------------------------ calibration
    def calibrate(self, xcal: torch.Tensor, residual: bool = False, stream=None) -> torch.Tensor:
        """Calibrate on xcal [B, T, d_model] (fp32, device); returns the layer output."""
        B, T, _ = xcal.shape
        ws = torch.empty(lib.calib_workspace_bytes(self.shape, B, T), dtype=torch.uint8,
                         device=self.device)
        out = torch.empty_like(xcal)
        lib.calibrate_layer(self.struct, self.conv_b, self.exps, self.conv_bq, self.static_amax,
                            xcal, B, T, int(residual), out, ws, stream)
        return out

    def exponents(self) -> dict:
        """Exponent table and static scales as numpy (for tests and reports)."""
        e = self.exps.cpu().numpy()
        X, s = self.layout, self.shape
        cc, nh = s.conv_ch, s.nheads
        amax = self.static_amax.cpu().numpy()
        return dict(e_u=e[X.e_u:X.e_u + cc], e_w=e[X.e_w:X.e_w + cc], e_o=e[X.e_o:X.e_o + cc],
                    e_x=e[X.e_x:X.e_x + nh], e_B=int(e[X.e_B]), e_C=int(e[X.e_C]),
                    e_h=e[X.e_h:X.e_h + nh], e_y=e[X.e_y:X.e_y + nh], e_D=e[X.e_D:X.e_D + nh],
                    e_g=int(e[X.e_g]), amax_in=float(amax[0]), amax_out=float(amax[1]),
                    conv_bq=self.conv_bq.cpu().numpy())

    # ------------------------------------------------------------ running
    def workspace(self, B: int, T: int) -> torch.Tensor:
        return torch.empty(lib.workspace_bytes(self.shape, B, T), dtype=torch.uint8,
                           device=self.device)

    def prefill(self, x: torch.Tensor, residual: bool = False, conv_state=None, ssm_state=None,
                out=None, ws=None, stream=None) -> torch.Tensor:
        B, T, _ = x.shape
        out = torch.empty_like(x) if out is None else out
        ws = self.workspace(B, T) if ws is None else ws
        lib.mixer_prefill(self.struct, x, B, T, int(residual), conv_state, ssm_state, out, ws,
                          stream)
        return out

    def decode(self, x: torch.Tensor, conv_state, ssm_state, residual: bool = False, out=None,
               ws=None, stream=None) -> torch.Tensor:
        B = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        ws = self.workspace(B, 1) if ws is None else ws
        lib.decode_step(self.struct, x, B, int(residual), conv_state, ssm_state, out, ws, stream)
        return out

    # ------------------------------------------------------------ FastMamba-LQ
    def lq_workspace(self, B: int, T: int) -> torch.Tensor:
        return torch.empty(lib.lq_workspace_bytes(self.shape, B, T), dtype=torch.uint8,
                           device=self.device)

    def lq_prefill(self, x: torch.Tensor, residual: bool = False, conv_state=None,
                   ssm_state=None, out=None, ws=None, stream=None) -> torch.Tensor:
        """The LQ variant of this layer: the same W8A8 linears and scales, the
        conv, scan and gate in fp32 (fp32 states from lq_new_states)."""
        B, T, _ = x.shape
        out = torch.empty_like(x) if out is None else out
        ws = self.lq_workspace(B, T) if ws is None else ws
        lib.lq_mixer_prefill(self.struct, self.lq_struct, x, B, T, int(residual), conv_state,
                             ssm_state, out, ws, stream)
        return out

    def lq_new_states(self, B: int):
        s = self.shape
        return (torch.zeros((B, 3, s.conv_ch), dtype=torch.float32, device=self.device),
                torch.zeros((B, s.nheads, s.headdim, s.d_state), dtype=torch.float32,
                            device=self.device))

    def new_states(self, B: int):
        s = self.shape
        sdt = torch.int16 if lib.STATE_BITS == 16 else torch.int32  # the state spec's storage
        return (torch.zeros((B, 3, s.conv_ch), dtype=torch.int8, device=self.device),
                torch.zeros((B, s.nheads, s.headdim, s.d_state), dtype=sdt, device=self.device))


class DeviceStack:
    """A stack of pre-normed residual mixer layers (no embedding / LM head)."""

    def __init__(self, layer_params: list, shape: MixerShape, rotate=1, mode=lib.FM_DYNAMIC,
                 device="cuda"):
        self.shape = shape
        self.layers = [DeviceLayer(p, shape, rotate, mode, prenorm=True, device=device)
                       for p in layer_params]

    def calibrate(self, xcal: torch.Tensor):
        r = xcal
        for L in self.layers:
            r = L.calibrate(r, residual=True)
        torch.cuda.synchronize()
        lib.sync_status()

    def prefill_(self, r: torch.Tensor, ws=None, states=None, stream=None) -> torch.Tensor:
        """In place: r <- r + mixer_l(RMSNorm(r)) for every layer."""
        B, T, _ = r.shape
        ws = self.layers[0].workspace(B, T) if ws is None else ws
        for i, L in enumerate(self.layers):
            cs, ss = states[i] if states is not None else (None, None)
            L.prefill(r, residual=True, conv_state=cs, ssm_state=ss, out=r, ws=ws, stream=stream)
        return r

    def stack_workspace(self, B: int, T: int, n_chunks: int) -> torch.Tensor:
        n = lib.stack_workspace_bytes(self.shape, len(self.layers), B, T, n_chunks)
        return torch.empty(n, dtype=torch.uint8, device=self.layers[0].device)

    def prefill_pipelined_(self, r: torch.Tensor, n_chunks: int = 2, ws=None, states=None,
                           stream=None) -> torch.Tensor:
        """As prefill_, in one fm_stack_prefill call: with n_chunks > 1 each
        sequence is cut into runs that pipeline through the layers on the
        library's own streams (bit-identical to prefill_)."""
        B, T, _ = r.shape
        ws = self.stack_workspace(B, T, n_chunks) if ws is None else ws
        lib.stack_prefill([L.struct for L in self.layers], r, B, T, states, n_chunks, ws, stream)
        return r

    def prefill_host(self, x_host: torch.Tensor, out_host: torch.Tensor, x_dev: torch.Tensor,
                     n_chunks: int = 2, ws=None, states=None, stream=None) -> torch.Tensor:
        """The stack on a batch in host memory (fm_stack_prefill_host): x_host in,
        out_host out (pinned host tensors), x_dev the device rows it runs in.
        Asynchronous on the stream: out_host is final after synchronising it."""
        B, T, _ = x_host.shape
        ws = self.stack_workspace(B, T, n_chunks) if ws is None else ws
        lib.stack_prefill_host([L.struct for L in self.layers], x_host, out_host, x_dev, B, T,
                               states, n_chunks, ws, stream)
        return out_host
