// What the tensor-core (tcgen05) path keeps per layer handle.
#pragma once

struct TcState {
  int enabled;
};
