"""B200-native (sm_100a) chunkwise mLSTM behind a C ABI: forward, backward and
the single-token step.

The computation runs in ``libmlstm_fw.so`` (hand-written CUDA kernels; see
``include/mlstm_fw.h``).  This package only builds that library
(``build.py``), marshals arguments into it (``api.py``) and draws seeded
synthetic inputs (``inputs.py``).
"""
from .api import (MlstmError, substep_workspace_size, last_device_error, mlstm_bw,  # noqa: F401
                  mlstm_bw_saved, mlstm_chunkwise, mlstm_fw, mlstm_fw_chunk_states,
                  mlstm_fw_parallel, mlstm_fw_train, mlstm_step, set_watchdog, train_sizes,
                  workspace_size)
