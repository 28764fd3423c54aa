"""B200-native (sm_100a) chunkwise mLSTM forward pass behind a C ABI.

The computation runs in ``libmlstm_fw.so`` (hand-written CUDA kernels; see
``include/mlstm_fw.h``).  This package only builds that library
(``build.py``), marshals arguments into it (``api.py``) and draws seeded
synthetic inputs (``inputs.py``).
"""
from .api import (MlstmError, substep_workspace_size, last_device_error, mlstm_fw,  # noqa: F401
                  mlstm_fw_chunk_states, mlstm_fw_parallel, set_watchdog, workspace_size)
